// halo_tc2.cuh -- stride-1 bf16 kernel for blocked local self-attention with
// haloing on sm_100a, organised around the tensor core's instruction rate.
//
// Operation (HaloNet, "Scaling Local Self-Attention for Parameter Efficient
// Visual Backbones", sections 2.1-2.2 and appendix A; index conventions of the
// blog page's RelPosEmb / HaloAttention modules):
//   z[q, key] = s * q . (k[key] + rel_h[kr - qy + w - 1] + rel_w[kc - qx + w - 1])
//   out[q]    = sum over in-image window keys of softmax(z) * v[key]
//
// On B200 a tcgen05.mma costs on the order of a hundred cycles of latency
// whatever its size below N = 128, and MMAs of one issuing thread run one
// after the other; only separate issuing threads overlap.  With dim_head 16
// or 32 the A.V product is a long chain of such small MMAs, so this kernel
// (a) packs two heads into every 128-row tile, (b) folds the relative dot
// products into the QK^T MMA as 56 extra B rows (N = 256), and (c) splits the
// A.V chain over the warps of the softmax warpgroup, each issuing its own
// K-step range into its own accumulator.
//
// Work item = one 8x8 query block and a pair of heads (a, b):
//   * TMA (warp 8): Q_a, Q_b [64 x d], K_a, K_b [w*w keys] and V_a, V_b; every
//     K tile is followed in shared memory by 4 zero rows and the 56-row
//     relative table R = [rel_h; 0; rel_w; 0] written once at start-up.
//   * S MMA (warp 9): S_h = Q_h [K_h; R]^T, M=64, N=256 into the TMEM lane half
//     of head h (lanes 0-15 of each quadrant for a, 16-31 for b), so TMEM lane
//     L holds one query row of one head: columns [0, w*w) are q.k, columns
//     [200, 256) the relative dot products q.rel_h[.] and q.rel_w[.].
//   * softmax warpgroup (one thread per TMEM lane = one query row): gather the
//     14 + 14 relative logits of its query, then the window keys in three
//     (d = 16) or two (d = 32) chunks of whole K-steps, each with its own
//     exact maximum; exponentials part on MUFU, part as a cubic polynomial on
//     the FMA pipe; bf16 P written back into the same TMEM lane (tcgen05.st)
//     over the consumed S columns.
//   * A.V (warp q of the warpgroup issues chunk q): O_q = P[:, keys of chunk q]
//     [V_a | V_b | 1], M=128 with P read from TMEM, N = 3d for d = 16 (the
//     ones block yields the chunk's row sum of the bf16 P) or N = 2d for
//     d = 32 (row sums added on the CUDA cores); head a's rows use the V_a
//     columns, head b's the V_b columns.
//   * epilogue: O = sum over chunks of 2^(c(m_q - m)) * O_q, divided by the
//     same combination of the chunk row sums, bf16, stored NHWC.
// Two softmax warpgroups work on alternate items, each in its own half of
// TMEM.  Every wait is bounded and reports HALO_ERR_TIMEOUT.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <utility>

#include "halo_tc.cuh"
#include "sm100.cuh"

namespace halo {
namespace tc2 {

using namespace sm100;
using tc::exp2_mufu;
using tc::pack_bf16x2;
using tc::record_timeout;
using tc::swz;

constexpr int kBlock = 8;
constexpr int kThreads = 384;     // warpgroups 0-1 softmax, warpgroup 2 producer (warp 8 TMA, 9 MMA)
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kSoftmaxRegs = tc::kSoftmaxRegs;
constexpr int kProducerRegs = tc::kProducerRegs;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlotCols = 256;   // one item per slot; warpgroup g owns slot g
constexpr int kKRows = 256;           // K tile: keys, zero pad up to row 200, R at [200, 256)
constexpr int kRBase = 200;           // first R row = first G column
constexpr int kRelW = 28;             // rel_w rows start at R row 28
constexpr int kScratchLine = 60;      // floats per thread of the gather scratch (56 used)
constexpr uint64_t kWaitNs = tc::kWaitNs;

struct Params {
  const __nv_bfloat16* rel_h;
  const __nv_bfloat16* rel_w;
  __nv_bfloat16* out;
  int N, H, W, heads, halo;
  int nbx, nby;
  int num_items;   // N * nby * nbx * heads / 2
  int stages;
  float c;         // log2(e) / sqrt(d)
};

template <int D, int WIN>
struct Cfg {
  static constexpr int ROWB = D * 2;
  static constexpr int KS = WIN * WIN;                    // window keys
  static constexpr int KSTEPS = (KS + 15) / 16;           // A.V K-steps
  static constexpr int KP = KSTEPS * 16;                  // keys incl. zero padding
  // The keys are cut into NCHUNK chunks of whole K-steps; each chunk has its
  // own row maximum and its own A.V accumulator, issued by its own warp.
  static constexpr int NCHUNK = (D == 16) ? 3 : 2;
  static constexpr int NSTREAM = NCHUNK;
  // d = 16: a third B atom of ones makes the A.V MMA also produce the row
  // sums of the bf16 P it consumed; d = 32 sums on the CUDA cores.
  static constexpr bool SUM_BY_MMA = (D == 16);
  static constexpr int PCOLS = KP / 2;                    // packed bf16 P columns in TMEM
  static constexpr int O_N = SUM_BY_MMA ? 3 * D : 2 * D;  // A.V N: [V_a | V_b (| ones)]
  static constexpr int O_BASE = (PCOLS + 7) / 8 * 8;      // first O column
  static constexpr int Q_TILE = 64 * ROWB;
  static constexpr int K_TILE = kKRows * ROWB;
  static constexpr int V_TILE = KP * ROWB;
  static constexpr int ONES_TILE = SUM_BY_MMA ? V_TILE : 0;  // right after V_b: third atom at 2*LBO
  static constexpr int STAGE_RAW = 2 * (Q_TILE + K_TILE + V_TILE) + ONES_TILE;
  static constexpr int STAGE_BYTES = (STAGE_RAW + 1023) / 1024 * 1024;
  static constexpr int TX_BYTES = 2 * (64 + 2 * KS) * ROWB;
  static constexpr int SCRATCH = 256 * kScratchLine * 4;
  static constexpr SmemSwizzle SW = (ROWB == 32) ? SW_32B : (ROWB == 64 ? SW_64B : SW_128B);
  static constexpr uint32_t SBO = 8 * ROWB;
  static constexpr int HALO = (WIN - kBlock) / 2;
  // exponentials taken by the polynomial: a subset of the block's own 8
  // columns [HALO, HALO+8), which are never outside the image
  static constexpr int NPOLY = (WIN * 2 + 2) / 5;
  static_assert(D == 16 || D == 32, "dim_head 16 or 32");
  static_assert(WIN % 2 == 0 && WIN >= 8 && WIN <= 14, "window 8..14");
  static_assert(KS <= kRBase, "S columns below the relative logits");
  static_assert(2 * WIN - 1 <= kRelW, "relative table rows");
  static_assert(O_BASE + NSTREAM * O_N <= (int)kSlotCols, "O accumulators in the slot");
  static_assert(NPOLY <= 8, "polynomial columns");
};

// First K-step of chunk i (i = 0..NCHUNK); chunk i covers keys
// [16*chunk_step(i), 16*chunk_step(i+1)), the last one ending at the window.
template <int KSTEPS, int NCHUNK>
__host__ __device__ constexpr int chunk_step(int i) {
  return (KSTEPS * i + NCHUNK / 2) / NCHUNK;
}

template <int D, int WIN>
__host__ __device__ constexpr int smem_bytes(int stages) {
  using C = Cfg<D, WIN>;
  return 1024 + C::SCRATCH + stages * C::STAGE_BYTES;
}

// Which window-column pairs (kc, kc+1), kc even, take the polynomial
// exponential: about 30% of the columns, inside the block's own 8 columns
// [h, h+8), which are never outside the image.  Bit kc/2 of the mask.
#ifndef HALO_TC2_POLY_PAIRS
#define HALO_TC2_POLY_PAIRS ((WIN * 3 + 10) / 20)  // 14 -> 2, 12 -> 2, 10 -> 2, 8 -> 1
#endif
template <int WIN>
__host__ __device__ constexpr unsigned poly_pair_mask(int npairs = HALO_TC2_POLY_PAIRS) {
  constexpr int h = (WIN - kBlock) / 2;
  unsigned m = 0;
  int picked = 0;
  // even kc inside [h, h+8) with kc+1 < h+8, from the middle outwards
  const int mid = (h + 3) & ~1;
  for (int d = 0; d < 8 && picked < npairs; ++d) {
    const int kc = mid + ((d & 1) ? -2 * ((d + 1) / 2) : 2 * (d / 2));
    if (kc >= h && kc + 1 < h + 8 && !((m >> (kc / 2)) & 1u)) {
      m |= 1u << (kc / 2);
      ++picked;
    }
  }
  return m;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x for a pair of x <= 0 with packed f32x2 arithmetic on the FMA pipe:
// x = j + f, j = floor(x) by a round-down add of 1.5*2^23 (adding it rounds
// to an integer), f in [0, 1); 2^f by a cubic fitted to the relative error
// on [0, 1) with p(0) = 1 (max relative error 8.6e-5); 2^j added into the
// exponent field.  x is clamped at -127, so masked (-inf) logits give
// exactly 0.  Returns the values' bit patterns.
__device__ __forceinline__ void exp2_poly2(float2 x, uint32_t& rx, uint32_t& ry) {
  x.x = fmaxf(x.x, -127.0f);
  x.y = fmaxf(x.y, -127.0f);
  const float2 t = __fadd2_rd(x, make_float2(12582912.0f, 12582912.0f));
  const float2 j = __fadd2_rn(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = __ffma2_rn(j, make_float2(-1.0f, -1.0f), x);
  float2 q = __ffma2_rn(f, make_float2(0.0770670548f, 0.0770670548f), make_float2(0.2276449651f, 0.2276449651f));
  q = __ffma2_rn(q, f, make_float2(0.6951168180f, 0.6951168180f));
  q = __ffma2_rn(q, f, make_float2(1.0f, 1.0f));
  rx = __float_as_uint(q.x) + (__float_as_uint(t.x) << 23);
  ry = __float_as_uint(q.y) + (__float_as_uint(t.y) << 23);
}

// bf16x2 of two floats given as bit patterns, round to nearest even: the
// P operand of the A.V MMA.  (Measured: truncating saves little and doubles
// the worst-case error of a P value; rounding with integer adds and a byte
// permute instead of the conversion instruction is slower, 117 against
// 111 us on the stage-1 workload.)
__device__ __forceinline__ uint32_t pack_p(uint32_t lo, uint32_t hi) {
  return pack_bf16x2(__uint_as_float(lo), __uint_as_float(hi));
}

// tcgen05.ld / st, 32 lanes x 32 bit: thread t <-> lane t of the warp's quadrant
__device__ __forceinline__ void tmem_ld_x32(uint32_t taddr, float* r) {
  uint32_t v[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) r[i] = __uint_as_float(v[i]);
}
__device__ __forceinline__ void tmem_ld_x8(uint32_t taddr, float* r) {
  uint32_t v[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 8; ++i) r[i] = __uint_as_float(v[i]);
}
// Load NC (a multiple of 8) consecutive columns starting at taddr.
template <int NC>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float* r) {
  static_assert(NC % 8 == 0, "columns in groups of 8");
#pragma unroll
  for (int i = 0; i + 32 <= NC; i += 32) tmem_ld_x32(taddr + i, r + i);
#pragma unroll
  for (int i = NC / 32 * 32; i < NC; i += 8) tmem_ld_x8(taddr + i, r + i);
}
__device__ __forceinline__ void tmem_st_x8(uint32_t taddr, const uint32_t* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

struct ItemCoord {
  int n, by, bx, pair;
};
__device__ __forceinline__ ItemCoord item_coord(int item, int pairs, int nbx, int nby) {
  ItemCoord c;
  c.pair = item % pairs;
  const int blk = item / pairs;
  c.bx = blk % nbx;
  c.by = (blk / nbx) % nby;
  c.n = blk / (nbx * nby);
  return c;
}

// Softmax of one chunk of window keys [J0, J1) of this thread's query row:
// z = S + rel_w (+ rel_h per window row), exact chunk maximum, exponentials,
// chunk row sum, packed bf16 P stored over TMEM columns [J0/2, JP/2) where JP
// pads the chunk to whole K-steps (keys >= J1 get P = 0).  Window rows have
// an even number of keys, so a packed pair never straddles two rows.
template <int WIN, int J0, int J1, int JP, bool SUM>
__device__ __forceinline__ void softmax_chunk(uint32_t ts, const float (&rw)[WIN], const float (&rh)[WIN], float c,
                                              float& m_out, float& l_out) {
  constexpr int NL = (J1 - J0 + 7) / 8 * 8;  // S columns loaded (multiple of 8)
  constexpr int NW = (JP - J0) / 2;          // packed P words
  constexpr int NP = (J1 - J0) / 2;          // key pairs of the chunk
  static_assert(J0 % 2 == 0 && J1 % 2 == 0 && WIN % 2 == 0 && NW % 8 == 0, "pairs never straddle rows");
  constexpr int R0 = J0 / WIN, NR = (J1 - 1) / WIN - R0 + 1;
  constexpr unsigned kPoly = poly_pair_mask<WIN>();
  float z[NL];
  tmem_ld_cols<NL>(ts + J0, z);
  tmem_wait_ld();
  // z = S + rel_w (pairs); per window row the maximum; chunk maximum of z + rel_h
  float2 zz[NP];
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    const int kc = (J0 + 2 * i) % WIN;
    zz[i] = __fadd2_rn(make_float2(z[2 * i], z[2 * i + 1]), make_float2(rw[kc], rw[kc + 1]));
  }
  float m = -INFINITY;
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    constexpr int dummy = 0;
    (void)dummy;
    const int i0 = ((R0 + r) * WIN > J0 ? (R0 + r) * WIN - J0 : 0) / 2;
    const int i1 = (((R0 + r) * WIN + WIN < J1 ? (R0 + r) * WIN + WIN : J1) - J0) / 2;
    float mr = -INFINITY;
#pragma unroll
    for (int i = i0; i < i1; ++i) mr = max3f(mr, zz[i].x, zz[i].y);
    m = fmaxf(m, mr + rh[R0 + r]);
  }
  // a chunk without in-image keys keeps m = -inf (weight 0 in the epilogue)
  // and takes its exponentials against 0: all of them are exactly 0
  const float mcr = (m == -INFINITY ? 0.f : m) * c;
  float brow[NR];  // per window row: c*rel_h - c*m; -inf outside the image
#pragma unroll
  for (int r = 0; r < NR; ++r) brow[r] = fmaf(rh[R0 + r], c, -mcr);
  // p = 2^(c*z - c*m); rows outside the image give exact 0
  float2 lacc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  uint32_t pk[NW];
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    const int j = J0 + 2 * i;
    const float bias = brow[j / WIN - R0];
    const float2 x = __ffma2_rn(zz[i], make_float2(c, c), make_float2(bias, bias));
    uint32_t rx, ry;
    if ((kPoly >> ((j % WIN) / 2)) & 1u) {
      exp2_poly2(x, rx, ry);
    } else {
      rx = __float_as_uint(exp2_mufu(x.x));
      ry = __float_as_uint(exp2_mufu(x.y));
    }
    if constexpr (SUM) lacc[i & 3] = __fadd2_rn(lacc[i & 3], make_float2(__uint_as_float(rx), __uint_as_float(ry)));
    pk[i] = pack_p(rx, ry);
  }
#pragma unroll
  for (int i = NP; i < NW; ++i) pk[i] = 0u;
#pragma unroll
  for (int i = 0; i < NW; i += 8) tmem_st_x8(ts + J0 / 2 + i, pk + i);
  const float2 la = __fadd2_rn(lacc[0], lacc[1]), lb = __fadd2_rn(lacc[2], lacc[3]);
  m_out = m;
  l_out = (la.x + lb.x) + (la.y + lb.y);
}

// All chunks of the row, in order (each with its own maximum).
template <int WIN, class C, int... I>
__device__ __forceinline__ void run_chunks(uint32_t ts, const float (&rw)[WIN], const float (&rh)[WIN], float c,
                                           float (&mch)[C::NCHUNK], float (&lch)[C::NCHUNK],
                                           std::integer_sequence<int, I...>) {
  (softmax_chunk<WIN, 16 * chunk_step<C::KSTEPS, C::NCHUNK>(I),
                 (I + 1 == C::NCHUNK) ? C::KS : 16 * chunk_step<C::KSTEPS, C::NCHUNK>(I + 1),
                 16 * chunk_step<C::KSTEPS, C::NCHUNK>(I + 1), !C::SUM_BY_MMA>(ts, rw, rh, c, mch[I], lch[I]),
   ...);
}

template <int D, int WIN>
__global__ void __launch_bounds__(kThreads, 1)
    halo_fwd_tc2(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                 const __grid_constant__ CUtensorMap tmap_v, const Params p) {
  using C = Cfg<D, WIN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* sScratch = reinterpret_cast<float*>(smem);             // 256 x 60 floats
  uint8_t* sStage = smem + (C::SCRATCH + 1023) / 1024 * 1024;   // stages x STAGE_BYTES
  // stage layout: [Q_a][Q_b][K_a][K_b][V_a][V_b][ones]
  constexpr int OFF_QA = 0, OFF_QB = C::Q_TILE;
  constexpr int OFF_KA = 2 * C::Q_TILE, OFF_KB = OFF_KA + C::K_TILE;
  constexpr int OFF_VA = OFF_KB + C::K_TILE, OFF_VB = OFF_VA + C::V_TILE;
  constexpr int OFF_ONES = OFF_VB + C::V_TILE;  // d = 16: ones atom of the A.V B operand

  __shared__ __align__(8) uint64_t bar_full[8];
  __shared__ __align__(8) uint64_t bar_empty[8];
  __shared__ __align__(8) uint64_t bar_sfull[2];
  __shared__ __align__(8) uint64_t bar_ofull[2];
  __shared__ __align__(8) uint64_t bar_tfree[2];
  __shared__ __align__(8) uint64_t bar_done[2];
  __shared__ __align__(8) uint64_t bar_pvdone[8];  // per softmax warp: its A.V MMAs finished
  __shared__ __align__(8) uint64_t bar_pready[2];  // per warpgroup: all four warps stored P
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
      mbar_init(&bar_empty[i], C::NSTREAM);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&bar_sfull[g], 1);
      mbar_init(&bar_ofull[g], C::NSTREAM);
      mbar_init(&bar_tfree[g], 4);
      mbar_init(&bar_pready[g], 4);
    }
    mbar_init(&bar_done[0], 1);
    mbar_init(&bar_done[1], 1);
    for (int w = 0; w < 8; ++w) mbar_init(&bar_pvdone[w], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kTmaWarp && lane == 0) {
    prefetch_tensormap(&tmap_q);
    prefetch_tensormap(&tmap_k);
    prefetch_tensormap(&tmap_v);
  }
  // Parts of every stage the TMA never writes: K tile rows [KS, 200) zero and
  // [200, 256) the relative table; V tile rows [KS, KP) zero.
  for (int s = 0; s < S; ++s) {
    uint8_t* st = sStage + s * C::STAGE_BYTES;
    for (int hb = 0; hb < 2; ++hb) {
      uint8_t* kt = st + (hb ? OFF_KB : OFF_KA);
      for (int idx = tid; idx < (kKRows - C::KS) * (D / 8); idx += kThreads) {
        const int r = C::KS + idx / (D / 8), u = idx % (D / 8);
        uint4 val = make_uint4(0, 0, 0, 0);
        const int rr = r - kRBase;
        if (rr >= 0 && rr < 2 * WIN - 1) val = *reinterpret_cast<const uint4*>(p.rel_h + rr * D + u * 8);
        else if (rr >= kRelW && rr < kRelW + 2 * WIN - 1)
          val = *reinterpret_cast<const uint4*>(p.rel_w + (rr - kRelW) * D + u * 8);
        *reinterpret_cast<uint4*>(kt + swz<C::ROWB>(r, u)) = val;
      }
      uint8_t* vt = st + (hb ? OFF_VB : OFF_VA);
      for (int idx = tid; idx < (C::KP - C::KS) * C::ROWB / 16; idx += kThreads)
        reinterpret_cast<uint4*>(vt + C::KS * C::ROWB)[idx] = make_uint4(0, 0, 0, 0);
    }
    if constexpr (C::SUM_BY_MMA) {
      for (int idx = tid; idx < C::ONES_TILE / 16; idx += kThreads)
        reinterpret_cast<uint4*>(st + OFF_ONES)[idx] = make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);
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

  const int pairs = p.heads / 2;
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
        const ItemCoord ic = item_coord(blockIdx.x + k * gridDim.x, pairs, p.nbx, p.nby);
        uint8_t* st = sStage + s * C::STAGE_BYTES;
        const int ha = 2 * ic.pair, x0 = ic.bx * kBlock, y0 = ic.by * kBlock;
        mbar_arrive_expect_tx(&bar_full[s], C::TX_BYTES);
        tma_load_4d(st + OFF_QA, &tmap_q, &bar_full[s], ha * D, x0, y0, ic.n);
        tma_load_4d(st + OFF_QB, &tmap_q, &bar_full[s], (ha + 1) * D, x0, y0, ic.n);
        tma_load_4d(st + OFF_KA, &tmap_k, &bar_full[s], ha * D, x0 - p.halo, y0 - p.halo, ic.n);
        tma_load_4d(st + OFF_KB, &tmap_k, &bar_full[s], (ha + 1) * D, x0 - p.halo, y0 - p.halo, ic.n);
        tma_load_4d(st + OFF_VA, &tmap_v, &bar_full[s], ha * D, x0 - p.halo, y0 - p.halo, ic.n);
        tma_load_4d(st + OFF_VB, &tmap_v, &bar_full[s], (ha + 1) * D, x0 - p.halo, y0 - p.halo, ic.n);
        issued = k + 1;
      }
      if (abort_flag) {
        for (int k = (issued > S ? issued - S : 0); k < issued; ++k)
          mbar_wait(&bar_full[k % S], (k / S) & 1, kWaitNs);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ S = Q [K; R]^T
    // (one issuing thread for both warpgroups, in item order: measured faster
    // than one issuing warp per warpgroup)
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(64, kKRows, false);
      for (int k = 0; k < my_items; ++k) {
        const int s = k % S, g = k & 1;
        if (!mbar_wait(&bar_full[s], (k / S) & 1, kWaitNs, &abort_flag)) {
          if (!abort_flag) record_timeout(&abort_flag);
          break;
        }
        if (k >= 2 && !mbar_wait(&bar_tfree[g], ((k >> 1) - 1) & 1, kWaitNs, &abort_flag)) {
          if (!abort_flag) record_timeout(&abort_flag);
          break;
        }
        tc_fence_after();
        const uint8_t* st = sStage + s * C::STAGE_BYTES;
        const uint32_t slot = tmem + g * kSlotCols;
#pragma unroll 1
        for (int hb = 0; hb < 2; ++hb) {
          const uint32_t qa = smem_addr(st + (hb ? OFF_QB : OFF_QA));
          const uint32_t ka = smem_addr(st + (hb ? OFF_KB : OFF_KA));
          const uint32_t dst = slot + (static_cast<uint32_t>(hb * 16) << 16);
          for (int ks = 0; ks < D / 16; ++ks)
            mma_f16_ss(dst, smem_desc(qa + 32 * ks, 16, C::SBO, C::SW), smem_desc(ka + 32 * ks, 16, C::SBO, C::SW),
                       idS, ks != 0);
        }
        mma_commit(&bar_sfull[g]);
      }
      mma_commit(&bar_done[0]);
      mbar_wait(&bar_done[0], 0, kWaitNs);
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
    const int hb = lane >> 4;            // 0: head a (lanes 0-15), 1: head b (lanes 16-31)
    const int row = 16 * wq + (lane & 15);  // query row in the 8x8 block
    const int qy = row >> 3, qx = row & 7;
    const uint32_t ts = tmem + g * kSlotCols + (static_cast<uint32_t>(32 * wq) << 16);
    float* line = sScratch + (g * 128 + wq * 32 + lane) * kScratchLine;
    const float c = p.c;
    const int C_all = p.heads * D;
    const uint32_t idO = idesc_bf16_f32(128, C::O_N, true);

    int j = 0;
    for (int k = g; k < my_items; k += 2, ++j) {
      if (!mbar_wait(&bar_sfull[g], j & 1, kWaitNs, &abort_flag)) {
        if (!abort_flag) record_timeout(&abort_flag);
        break;
      }
      tc_fence_after();
      const ItemCoord ic = item_coord(blockIdx.x + k * gridDim.x, pairs, p.nbx, p.nby);
      const int y0 = ic.by * kBlock - p.halo, x0 = ic.bx * kBlock - p.halo;

      // ---- relative logits of this query: G = TMEM columns [200, 256)
      float rh[WIN], rw[WIN];
      {
        float gv[56];
        tmem_ld_x32(ts + kRBase, gv);
        tmem_ld_x8(ts + kRBase + 32, gv + 32);
        tmem_ld_x8(ts + kRBase + 40, gv + 40);
        tmem_ld_x8(ts + kRBase + 48, gv + 48);
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 14; ++t)
          reinterpret_cast<float4*>(line)[t] = make_float4(gv[4 * t], gv[4 * t + 1], gv[4 * t + 2], gv[4 * t + 3]);
      }
#pragma unroll
      for (int kr = 0; kr < WIN; ++kr) {
        const int Y = y0 + kr;
        rh[kr] = (Y >= 0 && Y < p.H) ? line[kr - qy + WIN - 1] : -INFINITY;
      }
#pragma unroll
      for (int kc = 0; kc < WIN; ++kc) {
        const int X = x0 + kc;
        rw[kc] = (X >= 0 && X < p.W) ? line[kRelW + kc - qx + WIN - 1] : -INFINITY;
      }

      // ---- the key chunks: softmax, P into TMEM over the consumed S columns
      float mch[C::NCHUNK], lch[C::NCHUNK];
      run_chunks<WIN, C>(ts, rw, rh, c, mch, lch, std::make_integer_sequence<int, C::NCHUNK>{});
      tmem_wait_st();
      tc_fence_before();
      // the whole 128-row P is in TMEM before any A.V MMA reads it; a bounded
      // mbarrier (not bar.sync) so that a timeout elsewhere cannot deadlock
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_pready[g]);
      if (!mbar_wait(&bar_pready[g], j & 1, kWaitNs, &abort_flag)) {
        if (!abort_flag) record_timeout(&abort_flag);
        break;
      }
      tc_fence_after();

      // ---- A.V: warp w issues chunk w's K-steps (P from TMEM, V from shared memory)
      const int s = k % S;
      if (wq < C::NSTREAM && lane == 0) {
        const uint8_t* st = sStage + s * C::STAGE_BYTES;
        const uint32_t va = smem_addr(st + OFF_VA);
        const uint32_t slot = tmem + g * kSlotCols;
        const int kb = chunk_step<C::KSTEPS, C::NCHUNK>(wq), ke = chunk_step<C::KSTEPS, C::NCHUNK>(wq + 1);
        const uint32_t dst = slot + C::O_BASE + wq * C::O_N;
#pragma unroll 1
        for (int kk = kb; kk < ke; ++kk)
          mma_f16_ts(dst, slot + 8 * kk, smem_desc(va + kk * 16 * C::ROWB, C::V_TILE, C::SBO, C::SW), idO,
                     kk != kb);
        mma_commit(&bar_ofull[g]);
        mma_commit(&bar_empty[s]);
      }
      __syncwarp();

      // ---- epilogue: combine the chunk accumulators, normalise, store
      if (!mbar_wait(&bar_ofull[g], j & 1, kWaitNs, &abort_flag)) {
        if (!abort_flag) record_timeout(&abort_flag);
        break;
      }
      tc_fence_after();
      {
        // the whole warp loads every accumulator's columns (a warp-collective
        // load must not diverge; this thread's head is [0, D) for a, [D, 2D)
        // for b), then hands the slot back before the arithmetic and stores
        constexpr int kLd = C::SUM_BY_MMA ? 2 * D + 8 : 2 * D;  // one group of the ones columns
        float t[C::NCHUNK][kLd];
#pragma unroll
        for (int q = 0; q < C::NCHUNK; ++q) tmem_ld_cols<kLd>(ts + C::O_BASE + q * C::O_N, t[q]);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_tfree[g]);
        float mm = mch[0];
#pragma unroll
        for (int q = 1; q < C::NCHUNK; ++q) mm = fmaxf(mm, mch[q]);
        float o[D];
#pragma unroll
        for (int e = 0; e < D; ++e) o[e] = 0.f;
        float l = 0.f;
#pragma unroll
        for (int q = 0; q < C::NCHUNK; ++q) {
          const float f = exp2_mufu((mch[q] - mm) * c);
#pragma unroll
          for (int e = 0; e < D; ++e) o[e] = fmaf(f, hb ? t[q][D + e] : t[q][e], o[e]);
          // row sum of the bf16 P (ones columns) or of the fp32 exponentials
          if constexpr (C::SUM_BY_MMA) l = fmaf(f, t[q][kLd - 8], l);
          else l = fmaf(f, lch[q], l);
        }
        const float inv = 1.0f / l;
        uint32_t pk[D / 2];
#pragma unroll
        for (int t = 0; t < D / 2; ++t) pk[t] = pack_bf16x2(o[2 * t] * inv, o[2 * t + 1] * inv);
        const int head = 2 * ic.pair + hb;
        const int y = ic.by * kBlock + qy, x = ic.bx * kBlock + qx;
        __nv_bfloat16* dst = p.out + ((static_cast<size_t>(ic.n) * p.H + y) * p.W + x) * C_all + head * D;
#pragma unroll
        for (int t = 0; t < D / 8; ++t)
          reinterpret_cast<uint4*>(dst)[t] = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
      }
    }
    // A.V MMAs this warp issued are complete before TMEM is released
    if (lane == 0) {
      mma_commit(&bar_pvdone[warp]);
      mbar_wait(&bar_pvdone[warp], 0, kWaitNs);
    }
    __syncwarp();
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  named_bar_sync(1, kThreads);
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace tc2
}  // namespace halo
