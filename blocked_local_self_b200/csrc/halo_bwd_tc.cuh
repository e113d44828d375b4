// halo_bwd_tc.cuh -- tensor-core backward of blocked local self-attention with
// haloing on sm_100a: bf16, 8x8 query blocks, stride 1 or 2, dim_head 16 or 32,
// windows 8..14 (HaloNet, "Scaling Local Self-Attention for Parameter
// Efficient Visual Backbones", sections 2.1-2.2 and appendix A; the blog
// page's RelPosEmb / HaloAttention index conventions).
//
// Gradients of a loss L given dout = dL/dout.  Per query i and window key j,
// with p the softmax weights over the kept keys and s = d^-1/2:
//   dS_ij = p_ij (dout_i . v_j - dout_i . out_i)
//   dq = s (dS K + T R),  dk = s dS^T Q,  dv = P^T dout,  d[rel_h; rel_w] += s T^T Q
// where T (per query, one row of 64) holds the query's sums of dS over each
// window row at that row's rel_h table index and over each window column at
// that column's rel_w index, and R = [rel_h; 0; rel_w; 0] (64 rows).  All six
// products are tcgen05 MMAs.
//
// Work item = one 8x8 block of one head (stride 2: its 16 strided queries in
// rows 0-15 of the 64-row tiles; the sums over queries take those rows only,
// and the results of rows 16-63 are not used; the window is the stride-1
// one).  Two warpgroups take alternate items,
// each with a 256-column TMEM slot and its own P / dS / T buffers in shared
// memory; lane 0 of its warps issue its MMAs (independent chains in parallel):
//   R1  S = Q K^T (M=64, N=w^2 rounded to 8) at slot column 0 and
//       G = Q R^T (N=56) at column 200: the relative logits, gathered per
//       query as in the forward two-block kernel (out-of-image rows and
//       columns, and with the SASA mask of section 2.2 the rows and columns
//       outside the query's k x k square, get -inf).
//   softmax pass A: exact row maximum of c (S + rel); pass B: p' =
//       2^(c (S + rel) - m) as bf16 into the P buffer and the row sum l.
//   R2  dP = dout V^T (N as S) over the S columns, once every thread is done
//       with S.
//   pass C: p = p' / l, dS = p (dP - D) with D = dout . out (the forward's
//       output); bf16 p and dS into the P and dS buffers, the row and column
//       sums of dS into the query's T row.
//   R3  dV_t = P^T[keys of tile t] dout, dK_t = dS^T[tile t] Q (M=128, keys
//       in 128-row tiles), dQ = dS K + T R (M=64, two accumulators),
//       dR = T^T Q (M=64): four chains issued by the four warps.  One
//       shared-memory layout serves as the K-major A operand of dQ (rows =
//       queries, K = keys) and as the MN-major A operand of dK and dV
//       (M = keys, K = queries): rows of 64 keys (128 B, 128-byte swizzle),
//       atoms of 64 rows 8 KB apart.
//   epilogue: dk (x s) and dv of every in-image window key added to float32
//       accumulators in global memory (up to four windows hold a key); dq
//       (x s) stored as bf16; dR (x s) added to the warpgroup's table
//       accumulator in shared memory, flushed to global memory at exit.
// A TMA warp streams Q, dout, K and V (two stages when they fit).  Every wait
// is bounded and reports HALO_ERR_TIMEOUT.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <type_traits>

#include "halo_tc.cuh"
#include "halo_tc2.cuh"
#include "halo_tc4.cuh"
#include "sm100.cuh"

namespace halo {
namespace bwdtc {

using namespace sm100;
using tc::exp2_mufu;
using tc::pack_bf16x2;
using tc::record_timeout;
using tc::swz;
using tc2::tmem_ld_x8;
using tc4::tmem_ld_exact;

constexpr int kBlock = 8;
constexpr int kThreads = 288;        // warpgroups 0-1 (softmax, MMA issue), warp 8 TMA
constexpr int kTmaWarp = 8;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlotCols = 256;  // warpgroup g owns columns [256g, 256g + 256)
constexpr uint32_t kGBase = 200;     // G at slot columns [200, 256): rel_h logits, then rel_w at +28
constexpr int kRelW = 28;
constexpr int kRRows = 64;           // R tile rows: [rel_h; 0; rel_w; 0] padded to one 64-row K extent
constexpr uint64_t kWaitNs = tc::kWaitNs;

struct Params {
  const __nv_bfloat16* rel_h;
  const __nv_bfloat16* rel_w;
  const __nv_bfloat16* out;
  const __nv_bfloat16* dout;
  __nv_bfloat16* dq;
  float *dk32, *dv32, *drh32, *drw32;  // float32 accumulators (zeroed by the host)
  int N, H, W, heads, halo;
  int nbx, nby;
  int num_items;   // N * nby * nbx * heads
  int stages;
  int kmask;       // SASA mask size (0: none): keys within kmask/2 of the query
  float c;         // log2(e) / sqrt(d)
  float s;         // 1 / sqrt(d)
};

template <int D, int WIN, int STRIDE>
struct Cfg {
  static constexpr int ROWB = D * 2;
  static constexpr int QR = 64 / (STRIDE * STRIDE);    // query rows a block loads (Q and dout)
  static constexpr int KS = WIN * WIN;                 // window keys
  static constexpr int NS = (KS + 7) / 8 * 8;          // S / dP MMA N
  static constexpr int KP = (KS + 15) / 16 * 16;       // keys incl. padding: dQ K extent
  static constexpr int KSTEPS = KP / 16;
  static constexpr int MT = (KS + 127) / 128;          // 128-key tiles of dK / dV
  // Q and dout tiles: 64 rows at stride 1.  At stride 2 the QR = 16 loaded
  // rows only (1 KB): the M = 64 MMAs that take Q or dout as their A operand
  // (S, G, dP) read on into the next tile for rows 16-63, whose results are
  // never used, and the products summed over queries (dK, dV, dR) take one
  // K-step of 16 queries.  That halves the stage and fits two.
  static constexpr int Q_TILE = STRIDE == 1 ? 64 * ROWB : 1024;
  static constexpr int QKS = QR / 16;                  // K-steps over queries (dK, dV, dR)
  // A query row's keys are split between the two threads of its TMEM lane
  // (tcgen05.ld 16x32bx2): lanes 0-15 take window rows [0, R0), lanes 16-31
  // rows [R0, WIN), with K0 = R0 * WIN a multiple of 16 so that both halves
  // run NP pieces of 16 keys whose row / column indices are compile-time.
  static constexpr int R0 = (WIN == 8) ? 4 : 8;
  static constexpr int K0 = R0 * WIN;
  static constexpr int NP = K0 / 16;
  static_assert(K0 % 16 == 0 && KS - K0 <= K0 && R0 <= WIN, "key split");
  static_assert(QR * ROWB <= Q_TILE, "query rows in the tile");
  static constexpr int K_TILE = (KP * ROWB + 1023) / 1024 * 1024;
  static constexpr int OFF_Q = 0, OFF_DO = Q_TILE, OFF_K = 2 * Q_TILE, OFF_V = 2 * Q_TILE + K_TILE;
  static constexpr int STAGE_BYTES = 2 * Q_TILE + 2 * K_TILE;
  static constexpr int TX = (2 * QR + 2 * KS) * ROWB;
  static constexpr int R_TILE = (kRRows * ROWB + 1023) / 1024 * 1024;
  static constexpr int PBUF = MT * 2 * 8192;           // 64 queries x MT*128 keys, bf16, 8 KB atoms of 64 keys
  static constexpr int TBUF = 8192;                    // 64 queries x 64 table entries
  static constexpr int WG_BYTES = 2 * PBUF + TBUF;     // P, dS, T of one warpgroup
  static constexpr int DREL_BYTES = 2 * 64 * D * 4;    // two warpgroups' table accumulators (float32)
  // TMEM columns of R3's accumulators: dV tiles, dK tiles, dQ, dR
  // (after pass A the G columns are free too, so R3 may use the whole slot)
  static constexpr uint32_t COL_DV = 0, COL_DK = MT * D, COL_DQ = 2 * MT * D, COL_DQ2 = 2 * MT * D + D,
                            COL_DR = 2 * MT * D + 2 * D;
  static constexpr SmemSwizzle SW = (ROWB == 32) ? SW_32B : SW_64B;
  static constexpr uint32_t SBO = 8 * ROWB;
  static constexpr int HALO = (WIN - kBlock) / 2;
  static_assert(D == 16 || D == 32, "dim_head 16 or 32");
  static_assert(STRIDE == 1 || STRIDE == 2, "stride 1 or 2");
  static_assert(WIN % 2 == 0 && WIN >= 8 && WIN <= 14, "window 8..14");
  static_assert(NS <= (int)kGBase, "S columns below the relative logits");
  static_assert(COL_DR + D <= kSlotCols, "R3 accumulators in the slot");
  static_assert(2 * WIN - 1 <= kRelW && kRelW + 2 * WIN - 1 <= 56, "relative table rows");
};

template <int D, int WIN, int STRIDE>
__host__ __device__ constexpr int smem_bytes(int stages) {
  using C = Cfg<D, WIN, STRIDE>;
  return 1024 + C::R_TILE + 2 * C::WG_BYTES + C::DREL_BYTES + stages * C::STAGE_BYTES;
}

// tcgen05 instruction descriptor, kind::f16, bf16 A and B, f32 D, with the
// A major bit (15) as well as the B major bit (16).
__host__ __device__ constexpr uint32_t idesc_ab(int M, int N, bool a_mn, bool b_mn) {
  return idesc_bf16_f32(M, N, b_mn) | ((a_mn ? 1u : 0u) << 15);
}

// Byte offset of the 16-byte chunk holding keys [8u, 8u + 8) of query row r
// in a P / dS buffer: atoms of 64 keys (8 KB), 128-byte rows, 128-byte swizzle.
__device__ __forceinline__ uint32_t pofs(int r, int u) { return (u >> 3) * 8192 + swz<128>(r, u & 7); }

// A wait's outcome, the same for every lane of the warp (warp-collective
// tcgen05 instructions follow).
__device__ __forceinline__ bool warp_ok(bool ok) { return __all_sync(0xffffffffu, ok); }

// D consecutive TMEM columns of this thread's lane (32x32b shape).
template <int D>
__device__ __forceinline__ void tmem_ld_d(uint32_t taddr, float* r) {
  if constexpr (D == 32) tc2::tmem_ld_x32(taddr, r);
  else tmem_ld_exact<D>(taddr, r);
}

// A sweep over TMEM columns [0, NS) of this thread's lane in pieces of 16,
// the next piece's load in flight while the current one is processed:
// f(z, std::integral_constant<int, J0>) gets columns [J0, J0 + 16).
template <int J0, int NS, class F>
__device__ __forceinline__ void sweep16_at(uint32_t ts, uint32_t (&cur)[16], uint32_t (&nxt)[16], F& f) {
  if constexpr (J0 + 16 < NS) tmem_ld_32x32b_x16(ts + J0 + 16, nxt);
  float z[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) z[i] = __uint_as_float(cur[i]);
  f(z, std::integral_constant<int, J0>{});
  if constexpr (J0 + 16 < NS) {
    tmem_wait_ld();
    sweep16_at<J0 + 16, NS>(ts, nxt, cur, f);
  }
}
template <int NS, class F>
__device__ __forceinline__ void sweep16(uint32_t ts, F&& f) {
  uint32_t a[16], b[16];
  tmem_ld_32x32b_x16(ts, a);
  tmem_wait_ld();
  sweep16_at<0, NS>(ts, a, b, f);
}

// The same sweep over this thread's half of a row's keys: pieces [J0, J0 + 16)
// of keys K0 * half + J0 (lanes 16-31 read their partner's TMEM lane at
// column offset K0), for J0 < 16 * NP.
template <int J0, int NP, int K0, class F>
__device__ __forceinline__ void sweep_half_at(uint32_t ts, uint32_t (&cur)[16], uint32_t (&nxt)[16], F& f) {
  if constexpr (J0 + 16 < 16 * NP) tmem_ld_16x32bx2_x16<K0>(ts + J0 + 16, nxt);
  float z[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) z[i] = __uint_as_float(cur[i]);
  f(z, std::integral_constant<int, J0>{});
  if constexpr (J0 + 16 < 16 * NP) {
    tmem_wait_ld();
    sweep_half_at<J0 + 16, NP, K0>(ts, nxt, cur, f);
  }
}
template <int NP, int K0, class F>
__device__ __forceinline__ void sweep_half(uint32_t ts, F&& f) {
  uint32_t a[16], b[16];
  tmem_ld_16x32bx2_x16<K0>(ts, a);
  tmem_wait_ld();
  sweep_half_at<0, NP, K0>(ts, a, b, f);
}

// Barrier of one warpgroup's four warps on an mbarrier of count 4, so that
// the wait is bounded (a named barrier would hang if a warp gave up early).
// `ph` counts this warpgroup's uses of the barrier.
__device__ __forceinline__ bool wg_sync(uint64_t* bar, int& ph, int lane, int* abort_flag) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
  const bool ok = warp_ok(mbar_wait(bar, ph & 1, kWaitNs, abort_flag));
  ++ph;
  return ok;
}

template <int D, int WIN, int STRIDE>
__global__ void __launch_bounds__(kThreads, 1)
    halo_bwd_tc(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_do,
                const Params p) {
  using C = Cfg<D, WIN, STRIDE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sR = smem;
  uint8_t* sWG = sR + C::R_TILE;                          // [g][P | dS | T]
  float* sDrel = reinterpret_cast<float*>(sWG + 2 * C::WG_BYTES);  // [g][64][D]
  uint8_t* sStage = sWG + 2 * C::WG_BYTES + C::DREL_BYTES;

  // The stage of item k lands on bar_full[k % (2S)]: a barrier per stage and
  // per warpgroup, so that a warpgroup never waits on a barrier whose previous
  // phase (the other warpgroup's item k - S, at an odd stage count) is still
  // open, where a parity wait would pass one phase early.
  __shared__ __align__(8) uint64_t bar_full[8];
  __shared__ __align__(8) uint64_t bar_empty[4];
  __shared__ __align__(8) uint64_t bar_r1[2];
  __shared__ __align__(8) uint64_t bar_r2[2];
  __shared__ __align__(8) uint64_t bar_r3[2];
  __shared__ __align__(8) uint64_t bar_wg[2];    // count 4: the warps of warpgroup g
  __shared__ __align__(8) uint64_t bar_drain[8];  // per softmax warp (its lane 0 issues MMAs)
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int S = p.stages;

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_full[S + i], 1);
      mbar_init(&bar_empty[i], 4);   // the four R3 issuers
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&bar_r1[g], 2);      // S (warp 0) and G (warp 1)
      mbar_init(&bar_r2[g], 1);
      mbar_init(&bar_r3[g], 4);      // one commit per issuing warp
      mbar_init(&bar_wg[g], 4);
    }
    for (int w = 0; w < 8; ++w) mbar_init(&bar_drain[w], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kTmaWarp && lane == 0) {
    prefetch_tensormap(&tmap_q);
    prefetch_tensormap(&tmap_k);
    prefetch_tensormap(&tmap_v);
    prefetch_tensormap(&tmap_do);
  }
  // R tile, zeroed P / dS / T buffers and table accumulators, and the K / V
  // rows the TMA never writes
  for (int idx = tid; idx < kRRows * (D / 8); idx += kThreads) {
    const int r = idx / (D / 8), u = idx % (D / 8);
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r < 2 * WIN - 1) val = *reinterpret_cast<const uint4*>(p.rel_h + r * D + u * 8);
    else if (r >= kRelW && r < kRelW + 2 * WIN - 1)
      val = *reinterpret_cast<const uint4*>(p.rel_w + (r - kRelW) * D + u * 8);
    *reinterpret_cast<uint4*>(sR + swz<C::ROWB>(r, u)) = val;
  }
  for (int idx = tid; idx < (2 * C::WG_BYTES + C::DREL_BYTES) / 16; idx += kThreads)
    reinterpret_cast<uint4*>(sWG)[idx] = make_uint4(0, 0, 0, 0);
  for (int s = 0; s < S; ++s) {
    uint8_t* st = sStage + s * C::STAGE_BYTES;
    for (int idx = tid; idx < (C::KP - C::KS) * C::ROWB / 16; idx += kThreads) {
      reinterpret_cast<uint4*>(st + C::OFF_K + C::KS * C::ROWB)[idx] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(st + C::OFF_V + C::KS * C::ROWB)[idx] = make_uint4(0, 0, 0, 0);
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
  const int C_all = p.heads * D;

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
        const int item = blockIdx.x + k * gridDim.x;
        const int head = item % p.heads, blk = item / p.heads;
        const int bx = blk % p.nbx, by = (blk / p.nbx) % p.nby, n = blk / (p.nbx * p.nby);
        uint8_t* st = sStage + s * C::STAGE_BYTES;
        const int x0 = bx * kBlock, y0 = by * kBlock;
        uint64_t* full = &bar_full[k % (2 * S)];
        mbar_arrive_expect_tx(full, C::TX);
        tma_load_4d(st + C::OFF_Q, &tmap_q, full, head * D, x0, y0, n);
        tma_load_4d(st + C::OFF_DO, &tmap_do, full, head * D, x0 / STRIDE, y0 / STRIDE, n);
        tma_load_4d(st + C::OFF_K, &tmap_k, full, head * D, x0 - p.halo, y0 - p.halo, n);
        tma_load_4d(st + C::OFF_V, &tmap_v, full, head * D, x0 - p.halo, y0 - p.halo, n);
        issued = k + 1;
      }
      if (abort_flag) {
        for (int k = (issued > S ? issued - S : 0); k < issued; ++k)
          mbar_wait(&bar_full[k % (2 * S)], (k / (2 * S)) & 1, kWaitNs);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int g = warp >> 2;                 // warpgroup = TMEM slot
    const int wq = warp & 3;                 // lane quadrant
    const bool act = lane < 16;              // M=64 tiles: rows in lanes 0-15 of each quadrant
    const int row = 16 * wq + (lane & 15);   // query row in the 8x8 block (stride 2: rows 0-15)
    // rows with a query (stride 2: rows 0-15, warp 0); at stride 2 the other
    // rows' P, dS and T are written as zeros every item.  Both threads of a
    // TMEM lane work on its row (half = which part of its keys); `live`
    // marks the one that stores the row's dq.
    const bool rowlive = STRIDE == 1 || wq == 0;
    const bool live = act && rowlive;
    const int half = lane >> 4;
    const int qy = STRIDE == 1 ? (row >> 3) : 2 * ((row & 15) >> 2);
    const int qx = STRIDE == 1 ? (row & 7) : 2 * (row & 3);
    const uint32_t slot = tmem + g * kSlotCols;
    const uint32_t ts = slot + (static_cast<uint32_t>(32 * wq) << 16);
    uint8_t* sP = sWG + g * C::WG_BYTES;
    uint8_t* sDS = sP + C::PBUF;
    uint8_t* sT = sDS + C::PBUF;
    float* drel = sDrel + g * 64 * D;
    const bool elected = (wq == 0 && lane == 0);
    const float c = p.c;
    const uint32_t idS = idesc_ab(64, C::NS, false, false);
    const uint32_t idG = idesc_ab(64, 56, false, false);
    const uint32_t idKV = idesc_ab(128, D, true, true);   // dV, dK: A = P^T / dS^T (MN-major), B MN-major
    const uint32_t idQ = idesc_ab(64, D, false, true);    // dQ: A = dS / T (K-major), B MN-major
    const uint32_t idR = idesc_ab(64, D, true, true);     // dR: A = T^T (MN-major), B = Q (MN-major)
    const uint32_t pa = smem_addr(sP), dsa = smem_addr(sDS), tA = smem_addr(sT), ra = smem_addr(sR);
    int ph = 0;  // uses of bar_wg[g]

    bool ok = true;
    int j = 0;
    for (int k = g; k < my_items && ok; k += 2, ++j) {
      const int s = k % S;
      const uint8_t* st = sStage + s * C::STAGE_BYTES;
      const uint32_t qa = smem_addr(st + C::OFF_Q), doa = smem_addr(st + C::OFF_DO);
      const uint32_t ka = smem_addr(st + C::OFF_K), va = smem_addr(st + C::OFF_V);
      const int item = blockIdx.x + k * gridDim.x;
      const int head = item % p.heads, blk = item / p.heads;
      const int bx = blk % p.nbx, by = (blk / p.nbx) % p.nby, n = blk / (p.nbx * p.nby);
      const int y0 = by * kBlock - p.halo, x0 = bx * kBlock - p.halo;
      const int y = by * kBlock + qy, x = bx * kBlock + qx;
      const size_t pix = ((static_cast<size_t>(n) * p.H + y) * p.W + x) * C_all + static_cast<size_t>(head) * D;
      const int OH = p.H / STRIDE, OW = p.W / STRIDE;
      const size_t opix = ((static_cast<size_t>(n) * OH + y / STRIDE) * OW + x / STRIDE) * C_all +
                          static_cast<size_t>(head) * D;
      // this query's out and dout rows (for D = dout . out), in flight during the MMAs and pass A
      uint4 orow[D / 8], drow[D / 8];
#pragma unroll
      for (int e = 0; e < D / 8; ++e) {
        orow[e] = rowlive ? *reinterpret_cast<const uint4*>(p.out + opix + 8 * e) : make_uint4(0, 0, 0, 0);
        drow[e] = rowlive ? *reinterpret_cast<const uint4*>(p.dout + opix + 8 * e) : make_uint4(0, 0, 0, 0);
      }
      // ---- R1: S (warp 0) and G (warp 1), issued in parallel
      if (wq < 2 && lane == 0) {
        if (mbar_wait(&bar_full[k % (2 * S)], (k / (2 * S)) & 1, kWaitNs, &abort_flag)) {
          tc_fence_after();
          const uint32_t dst = slot + (wq ? kGBase : 0u), ba = wq ? ra : ka;
          const uint32_t id = wq ? idG : idS;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            mma_f16_ss(dst, smem_desc(qa + 32 * ks, 16, C::SBO, C::SW), smem_desc(ba + 32 * ks, 16, C::SBO, C::SW),
                       id, ks != 0);
          mma_commit(&bar_r1[g]);
        } else if (!abort_flag) {
          record_timeout(&abort_flag);
        }
      }
      ok = warp_ok(mbar_wait(&bar_r1[g], j & 1, kWaitNs, &abort_flag));
      if (!ok) break;
      tc_fence_after();

      // ---- relative logits of this query (log2 units), -inf for masked rows / columns
      float rh[WIN], rw[WIN];
      {
        float gh[WIN + 7];
        if constexpr (STRIDE == 1) {
          tmem_ld_exact<WIN + 1>(ts + kGBase + (WIN - 2 - 2 * wq), gh);
        } else {
          tmem_ld_exact<WIN + 7>(ts + kGBase + WIN - 8, gh);
        }
        float a[WIN + 7];
        tmem_ld_exact<WIN + 7>(ts + kGBase + kRelW + WIN - 8, a);
        tmem_wait_ld();
        if constexpr (STRIDE == 2) {
          // columns WIN - 8 + i: the query's entry kr - qy + WIN - 1 is i = kr + 7 - qy
          const int shh = 7 - qy;
#pragma unroll
          for (int i = 0; i < WIN + 3; ++i) gh[i] = (shh & 4) ? gh[i + 4] : gh[i];
#pragma unroll
          for (int i = 0; i < WIN + 1; ++i) gh[i] = (shh & 2) ? gh[i + 2] : gh[i];
#pragma unroll
          for (int i = 0; i < WIN; ++i) gh[i] = (shh & 1) ? gh[i + 1] : gh[i];
        }
        const bool odd = ((lane >> 3) & 1) != 0;
#pragma unroll
        for (int kr = 0; kr < WIN; ++kr) {
          const int Y = y0 + kr;
          const bool keep = Y >= 0 && Y < p.H &&
                            (p.kmask == 0 || (kr - qy - p.halo <= (p.kmask >> 1) && qy + p.halo - kr <= (p.kmask >> 1)));
          const float gv = STRIDE == 1 ? (odd ? gh[kr] : gh[kr + 1]) : gh[kr];
          rh[kr] = keep ? gv * c : -INFINITY;
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
          const bool keep = X >= 0 && X < p.W &&
                            (p.kmask == 0 || (kc - qx - p.halo <= (p.kmask >> 1) && qx + p.halo - kc <= (p.kmask >> 1)));
          rw[kc] = keep ? a[kc] * c : -INFINITY;
        }
      }
      // lanes 16-31 take their partner's (lanes 0-15 hold the row's TMEM lane)
#pragma unroll
      for (int i = 0; i < WIN; ++i) {
        rh[i] = __shfl_sync(0xffffffffu, rh[i], lane & 15);
        rw[i] = __shfl_sync(0xffffffffu, rw[i], lane & 15);
      }
      // this half's window rows: local row r is row r + R0 * half, -inf past the window
      float rhl[C::R0];
#pragma unroll
      for (int r = 0; r < C::R0; ++r) rhl[r] = half ? (r + C::R0 < WIN ? rh[(r + C::R0) % WIN] : -INFINITY) : rh[r];
      // ---- pass A: exact row maximum, per window row max of c S + c rel_w,
      // then over rows with c rel_h added (keys past the window: rhl = -inf)
      float m = -INFINITY;
      {
        float rmax[C::R0];
#pragma unroll
        for (int r = 0; r < C::R0; ++r) rmax[r] = -INFINITY;
        sweep_half<C::NP, C::K0>(ts, [&](const float (&z)[16], auto jc) {
          constexpr int J0 = decltype(jc)::value;
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            // keys past the window in the upper half: their columns may hold stale TMEM
            const bool tail = half && (J0 + t >= C::KS - C::K0);
            if (!tail) rmax[(J0 + t) / WIN] = fmaxf(rmax[(J0 + t) / WIN], fmaf(z[t], c, rw[(J0 + t) % WIN]));
          }
        });
#pragma unroll
        for (int r = 0; r < C::R0; ++r) m = fmaxf(m, rmax[r] + rhl[r]);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
      }
      // ---- D = dout . out of this query
      float Dq = 0.f;
#pragma unroll
      for (int e = 0; e < D / 8; ++e) {
        const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&orow[e]);
        const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&drow[e]);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float2 of = __bfloat1622float2(o2[t]), df = __bfloat1622float2(d2[t]);
          Dq = fmaf(of.x, df.x, fmaf(of.y, df.y, Dq));
        }
      }
      // ---- pass B: p' = 2^(c S + c rel_w + (c rel_h - m)) into the P buffer, row sum
      float brow[C::R0];
#pragma unroll
      for (int r = 0; r < C::R0; ++r) brow[r] = rhl[r] - m;
      // this half's first 8-key chunk of the P / dS rows; chunks past the
      // buffer (keys beyond MT * 128, all outside the window) are not stored
      const int u0 = half * (C::K0 / 8);
      float l = 0.f;
      sweep_half<C::NP, C::K0>(ts, [&](const float (&z)[16], auto jc) {
        constexpr int J0 = decltype(jc)::value;
        uint32_t pk[8];
#pragma unroll
        for (int t = 0; t < 16; t += 2) {
          const bool tail0 = half && (J0 + t >= C::KS - C::K0), tail1 = half && (J0 + t + 1 >= C::KS - C::K0);
          const float e0 = tail0 ? 0.f : exp2_mufu(fmaf(z[t], c, rw[(J0 + t) % WIN]) + brow[(J0 + t) / WIN]);
          const float e1 =
              tail1 ? 0.f : exp2_mufu(fmaf(z[t + 1], c, rw[(J0 + t + 1) % WIN]) + brow[(J0 + t + 1) / WIN]);
          l += e0 + e1;
          pk[t / 2] = pack_bf16x2(e0, e1);
        }
        if (!rowlive) {
#pragma unroll
          for (int t = 0; t < 8; ++t) pk[t] = 0u;
        }
        if (u0 + J0 / 8 < C::MT * 16) {
          *reinterpret_cast<uint4*>(sP + pofs(row, u0 + J0 / 8)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(sP + pofs(row, u0 + J0 / 8 + 1)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      });
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      const float inv_l = 1.0f / l;
      // ---- R2: dP = dout V^T over the S columns
      tc_fence_before();
      ok = wg_sync(&bar_wg[g], ph, lane, &abort_flag);
      if (!ok) break;
      if (elected) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_f16_ss(slot, smem_desc(doa + 32 * ks, 16, C::SBO, C::SW), smem_desc(va + 32 * ks, 16, C::SBO, C::SW),
                     idS, ks != 0);
        mma_commit(&bar_r2[g]);
      }
      ok = warp_ok(mbar_wait(&bar_r2[g], j & 1, kWaitNs, &abort_flag));
      if (!ok) break;
      tc_fence_after();
      // ---- pass C: p = p' / l, dS = p (dP - D); bf16 P and dS; row / column sums of dS
      // (keys past the window have p = 0, hence dS = 0)
      float rs[C::R0], cs[WIN];
#pragma unroll
      for (int i = 0; i < C::R0; ++i) rs[i] = 0.f;
#pragma unroll
      for (int i = 0; i < WIN; ++i) cs[i] = 0.f;
      sweep_half<C::NP, C::K0>(ts, [&](const float (&dp)[16], auto jc) {
        constexpr int J0 = decltype(jc)::value;
        const bool stored = u0 + J0 / 8 < C::MT * 16;
        uint4 pv[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
        if (stored) {
          pv[0] = *reinterpret_cast<const uint4*>(sP + pofs(row, u0 + J0 / 8));
          pv[1] = *reinterpret_cast<const uint4*>(sP + pofs(row, u0 + J0 / 8 + 1));
        }
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(pv);
        uint32_t pk[8], dk[8];
#pragma unroll
        for (int t = 0; t < 16; t += 2) {
          const float2 pp = __bfloat1622float2(p2[t / 2]);
          const float p0 = pp.x * inv_l, p1 = pp.y * inv_l;
          const bool tail0 = half && (J0 + t >= C::KS - C::K0), tail1 = half && (J0 + t + 1 >= C::KS - C::K0);
          const float d0 = tail0 ? 0.f : p0 * (dp[t] - Dq), d1 = tail1 ? 0.f : p1 * (dp[t + 1] - Dq);
          rs[(J0 + t) / WIN] += d0;
          cs[(J0 + t) % WIN] += d0;
          rs[(J0 + t + 1) / WIN] += d1;
          cs[(J0 + t + 1) % WIN] += d1;
          pk[t / 2] = pack_bf16x2(p0, p1);
          dk[t / 2] = pack_bf16x2(d0, d1);
        }
        if (!rowlive) {
#pragma unroll
          for (int t = 0; t < 8; ++t) pk[t] = dk[t] = 0u;
        }
        if (stored) {
          *reinterpret_cast<uint4*>(sP + pofs(row, u0 + J0 / 8)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(sP + pofs(row, u0 + J0 / 8 + 1)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          *reinterpret_cast<uint4*>(sDS + pofs(row, u0 + J0 / 8)) = make_uint4(dk[0], dk[1], dk[2], dk[3]);
          *reinterpret_cast<uint4*>(sDS + pofs(row, u0 + J0 / 8 + 1)) = make_uint4(dk[4], dk[5], dk[6], dk[7]);
        }
      });
#pragma unroll
      for (int i = 0; i < WIN; ++i) cs[i] += __shfl_xor_sync(0xffffffffu, cs[i], 16);
      // T row: rel_h entries kr - qy + w - 1 (each half its window rows),
      // rel_w entries 28 + kc - qx + w - 1 (lanes 0-15)
      if (act) {
#pragma unroll
        for (int u = 0; u < 8; ++u) *reinterpret_cast<uint4*>(sT + swz<128>(row, u)) = make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
      if (rowlive) {
#pragma unroll
        for (int i = 0; i < C::R0; ++i) {
          const int kr = i + C::R0 * half;
          if (kr < WIN) {
            const int ah = kr - qy + WIN - 1;
            *reinterpret_cast<__nv_bfloat16*>(sT + swz<128>(row, ah >> 3) + (ah & 7) * 2) = __float2bfloat16_rn(rs[i]);
          }
        }
        if (act) {
#pragma unroll
          for (int i = 0; i < WIN; ++i) {
            const int aw = kRelW + i - qx + WIN - 1;
            *reinterpret_cast<__nv_bfloat16*>(sT + swz<128>(row, aw >> 3) + (aw & 7) * 2) = __float2bfloat16_rn(cs[i]);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      ok = wg_sync(&bar_wg[g], ph, lane, &abort_flag);
      if (!ok) break;
      // ---- R3, four independent MMA chains on the four warps' lane 0:
      // warp 0 dV tiles, warp 1 dK tiles, warp 2 dQ = dS K, warp 3 T R (a
      // second dQ accumulator) and dR = T^T Q
      if (lane == 0) {
        tc_fence_after();
        if (wq < 2) {
          const uint32_t col = wq ? C::COL_DK : C::COL_DV;
          const uint32_t aa = wq ? dsa : pa, bb = wq ? qa : doa;
#pragma unroll 1
          for (int t = 0; t < C::MT; ++t)
#pragma unroll 1
            for (int ks = 0; ks < C::QKS; ++ks)
              mma_f16_ss(slot + col + t * D, smem_desc(aa + t * 16384 + ks * 2048, 8192, 1024, SW_128B),
                         smem_desc(bb + ks * 16 * C::ROWB, 16, C::SBO, C::SW), idKV, ks != 0);
        } else if (wq == 2) {
#pragma unroll 1
          for (int ks = 0; ks < C::KSTEPS; ++ks)
            mma_f16_ss(slot + C::COL_DQ, smem_desc(dsa + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024, SW_128B),
                       smem_desc(ka + ks * 16 * C::ROWB, 16, C::SBO, C::SW), idQ, ks != 0);
        } else {
#pragma unroll 1
          for (int ks = 0; ks < 4; ++ks) {
            mma_f16_ss(slot + C::COL_DQ2, smem_desc(tA + ks * 32, 16, 1024, SW_128B),
                       smem_desc(ra + ks * 16 * C::ROWB, 16, C::SBO, C::SW), idQ, ks != 0);
            if (ks < C::QKS)
              mma_f16_ss(slot + C::COL_DR, smem_desc(tA + ks * 2048, 8192, 1024, SW_128B),
                         smem_desc(qa + ks * 16 * C::ROWB, 16, C::SBO, C::SW), idR, ks != 0);
          }
        }
        mma_commit(&bar_r3[g]);
        mma_commit(&bar_empty[s]);
      }
      ok = warp_ok(mbar_wait(&bar_r3[g], j & 1, kWaitNs, &abort_flag));
      if (!ok) break;
      tc_fence_after();
      // ---- epilogue
#pragma unroll
      for (int t = 0; t < C::MT; ++t) {
        float dv[D], dk[D];
        tmem_ld_d<D>(ts + C::COL_DV + t * D, dv);
        tmem_ld_d<D>(ts + C::COL_DK + t * D, dk);
        tmem_wait_ld();
        const int key = t * 128 + 32 * wq + lane;
        const int kr = key / WIN, kc = key - (key / WIN) * WIN;
        const int Y = y0 + kr, X = x0 + kc;
        if (key < C::KS && Y >= 0 && Y < p.H && X >= 0 && X < p.W) {
          const size_t off = ((static_cast<size_t>(n) * p.H + Y) * p.W + X) * C_all + static_cast<size_t>(head) * D;
#pragma unroll
          for (int e = 0; e < D; e += 4) {
            atomicAdd(reinterpret_cast<float4*>(p.dv32 + off + e), make_float4(dv[e], dv[e + 1], dv[e + 2], dv[e + 3]));
            atomicAdd(reinterpret_cast<float4*>(p.dk32 + off + e),
                      make_float4(p.s * dk[e], p.s * dk[e + 1], p.s * dk[e + 2], p.s * dk[e + 3]));
          }
        }
      }
      {
        float dqv[D], drv[D];
        tmem_ld_d<D>(ts + C::COL_DQ, dqv);
        tmem_ld_d<D>(ts + C::COL_DR, drv);
        tmem_wait_ld();
        {
          float dq2[D];
          tmem_ld_d<D>(ts + C::COL_DQ2, dq2);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < D; ++e) dqv[e] += dq2[e];
        }
        if (live) {
          uint32_t pk[D / 2];
#pragma unroll
          for (int e = 0; e < D / 2; ++e) pk[e] = pack_bf16x2(p.s * dqv[2 * e], p.s * dqv[2 * e + 1]);
#pragma unroll
          for (int e = 0; e < D / 8; ++e)
            reinterpret_cast<uint4*>(p.dq + pix)[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
        if (act) {
          // dR row = table entry `row` (rows 56..63 stay zero)
#pragma unroll
          for (int e = 0; e < D; ++e) drel[row * D + e] += p.s * drv[e];
        }
      }
      tc_fence_before();
      ok = wg_sync(&bar_wg[g], ph, lane, &abort_flag);
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
  __syncthreads();
  tc_fence_after();
  // both warpgroups' table sums into the float32 accumulators
  for (int idx = tid; idx < (4 * WIN - 2) * D; idx += kThreads) {
    const int r = idx / D, e = idx % D;      // r < 2w - 1: rel_h row; 2w - 1 <= r: rel_w row r - (2w - 1)
    if (r < 2 * WIN - 1) {
      atomicAdd(p.drh32 + r * D + e, sDrel[r * D + e] + sDrel[64 * D + r * D + e]);
    } else if (r < 4 * WIN - 2) {
      const int rr = r - (2 * WIN - 1);
      atomicAdd(p.drw32 + rr * D + e, sDrel[(kRelW + rr) * D + e] + sDrel[64 * D + (kRelW + rr) * D + e]);
    }
  }
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace bwdtc
}  // namespace halo
