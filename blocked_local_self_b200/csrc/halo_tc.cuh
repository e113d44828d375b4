// halo_tc.cuh -- fused bf16 blocked local self-attention with haloing for
// sm_100a: TMA window loads, tcgen05 tensor-core QK^T / relative logits / PV
// with TMEM accumulators, masked softmax on the CUDA cores.
//
// Operation (HaloNet, "Scaling Local Self-Attention for Parameter Efficient
// Visual Backbones", sections 2.1-2.2 and appendix A; index conventions of the
// blog page's RelPosEmb / HaloAttention modules):
//   z[q, key] = s * q . (k[key] + rel_h[kr - qy + w - 1] + rel_w[kc - qx + w - 1])
//   out[q]    = sum over in-image window keys of softmax(z) * v[key]
//
// Design (one CTA per SM, persistent over work items):
//   * item = one 8x8 query block and one head (stride 1: 64 query rows), or
//     one block and PARTS heads (stride 2: 16 query rows per head, head p in
//     rows 16p..16p+15 of a 64-row MMA tile).
//   * warp 8 (one lane) streams items with TMA: the query tile and, per head,
//     the w x 16 window of K and of V (w = 8 + 2*halo rows; the window row is
//     padded from w to 16 keys so every window row is one 32-byte swizzle
//     chunk of the P operand).  Keys outside the image arrive as zeros.
//     Q and K travel on their own stage barrier, one item ahead of V, and
//     are released as soon as the S and G MMAs finish.
//   * warp 9 (one lane) issues S = Q K^T (tcgen05.mma, M=64, bf16 in, f32 in
//     TMEM) and warp 10 G = Q R^T with R = [rel_h; rel_w] (the 2(2w-1)
//     relative dot products of every query); after the softmax, warps
//     q < NST of the owning warpgroup each issue a share of O = P V (window
//     rows of one head) into their own accumulator, summed in the epilogue
//     (for d = 16 the row sums come from a ones tile appended to V).
//   * four heads of d = 32 per tile (stride 2) go in pairs: q, k, v boxes of
//     two heads (128-byte rows), Q/K barriers per pair, one A.V chain over
//     both pair tiles, P in TMEM (A operand of a TMEM-A MMA) and the shared
//     memory of the P tiles used as a second V buffer.
//   * warps 0-3 and 4-7 are two softmax warpgroups that take alternate items;
//     each owns one half of every TMEM lane quadrant (lanes 0-15 or 16-31), so
//     the MMAs of one item overlap the softmax of the other.  A query row is
//     split over two threads (tcgen05.ld 16x32bx2): the thread with lane < 16
//     takes the even window rows, its partner the odd ones.
//   * per row: gather the relative logits that apply to this query from G,
//     add them, mask out-of-image keys, exact row max, exponentials (part on
//     the MUFU unit), bf16 P into shared memory (or TMEM), then normalise O
//     and store bf16 NHWC directly.
//   Nothing but q, k, v, the tables and out touches global memory.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace halo {

__device__ int g_halo_error;  // sticky device error flag (HALO_ERR_TIMEOUT)

namespace tc {

using namespace sm100;

constexpr int kBlock = 8;         // query block side handled by this kernel
constexpr int kRowKeys = 16;      // P / V window row pitch in keys (w padded to 16)
constexpr int kThreads = 384;     // 2 softmax warpgroups + 1 producer warpgroup
constexpr int kTmaWarp = 8;       // producer warpgroup: warp 8 TMA, warps 9-10 MMA,
constexpr int kMmaWarp = 9;       // warp 11 idle
// Register split (setmaxnreg): the kernel launches with kLaunchRegs per thread
// (3 warps per SM sub-partition cap it at 168); the producer warpgroup gives
// registers back and the softmax warpgroups take more.  The sum stays within
// the launch allocation: 256*208 + 128*72 = 62464 <= 384*168 = 64512.
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 208;
constexpr int kProducerRegs = 72;
static_assert(256 * kSoftmaxRegs + 128 * kProducerRegs <= kThreads * kLaunchRegs, "register split");
// TMEM: 512 columns x 128 lanes.  Warpgroup g owns lanes 16g..16g+15 of every
// 32-lane quadrant (the two M=64 accumulator halves) and, inside that, two
// item slots of 256 columns: S at [0, 200), G at [200, 256); O (and the row
// sums) overwrite the first S columns once P has been taken from S.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlotCols = 256;
constexpr uint32_t kTmemG = 200;
constexpr int kGCols = 56;        // rel_h logits at [0, 2w-1), rel_w logits at [28, 28+2w-1)
constexpr int kGRelW = 28;
constexpr uint64_t kWaitNs = 1000000000ull;  // 1 s bound on every wait

struct Params {
  const __nv_bfloat16* rel_h;
  const __nv_bfloat16* rel_w;
  __nv_bfloat16* out;
  int N, H, W, heads, halo;
  int nbx, nby;            // blocks along x and y
  int num_items;           // total work items
  int heads_per_item;      // PARTS
  int stages;              // TMA pipeline depth
  int OH, OW;
  float c;                 // log2(e) / sqrt(d)
};

// PP = PARTS: heads per item at stride 2 (4 x 16 queries fill the 64-row
// tile; 2 at d = 32 when the head count is not a multiple of 4, 1 at d = 64).
template <int D, int WIN, int STRIDE, int PP>
struct Cfg {
  static constexpr int ROWB = D * 2;                      // bytes of one pixel's head slice
  static constexpr int PARTS = PP;
  static_assert(STRIDE == 2 || PP == 1, "one head per item at stride 1");
  static constexpr int QROWS_PER_HEAD = (STRIDE == 1) ? 64 : 16;
  // Four heads of d = 32 travel in pairs: one TMA box of 2d channels (128-byte
  // rows, 128B swizzle) per pair for q, k and v, half the box rows of one box
  // per head (the TMA unit's cost goes by rows).  A head's K-major operands
  // then start d*2 bytes into the row for the second head of a pair.
  static constexpr bool PAIRED = (STRIDE == 2 && PARTS == 4 && D == 32);
  static constexpr int HPB = PAIRED ? 2 : 1;              // heads per TMA box
  static constexpr int BOXES = PARTS / HPB;
  static constexpr int BROWB = ROWB * HPB;                // bytes of one pixel's row in a q/k/v tile
  // stride 1: 64-row Q tile.  stride 2: zero-gap buffer so that the 64-row view
  // of head p holds its 16 queries in rows 16p..16p+15 and zeros elsewhere
  // (paired: rows [16 zero][pair 0][48 zero][pair 1][16 zero], the views of
  // the two heads of a pair 16 rows apart).
  static constexpr int QBUF_ROWS = (STRIDE == 1) ? 64 : (PAIRED ? 112 : (112 + 48 * (PARTS - 1)));
  // buffer row of box b's first query, first buffer row of head p's view and
  // the byte offset of head p's channels in a row
  __host__ __device__ static constexpr int q_row(int b) { return PAIRED ? 16 + 64 * b : 48 + 64 * b; }
  __host__ __device__ static constexpr int view_row(int p) { return PAIRED ? q_row(p / 2) - 16 * p : 48 + 48 * p; }
  __host__ __device__ static constexpr int koff(int p) { return ROWB * (p % HPB); }
  static constexpr int KS = WIN * WIN;                    // keys of the window (K tile rows written)
  static constexpr int NS = (KS + 7) / 8 * 8;             // S columns (QK^T N); rows KS..NS-1 zero
  static constexpr int KP = WIN * kRowKeys;               // PV K extent (V tile rows, P columns)
  static constexpr int K_TILE = NS * BROWB;               // one box's K tile
  static constexpr int V_TILE = KP * BROWB;
  static constexpr int Q_BYTES = QBUF_ROWS * BROWB;
  // Paired heads keep P in TMEM (bf16 over the first S columns, the A operand
  // of a TMEM-A MMA), and the shared memory the P tiles took holds a second V
  // buffer: a stage is [Q | K of every box] then VPS V buffers, so the V of
  // item k + 1 loads while the A.V of item k runs.
  static constexpr int VPS = PAIRED ? 2 : 1;              // V buffers per stage
  static constexpr int QK_BYTES = Q_BYTES + BOXES * K_TILE;
  static constexpr int VB_BYTES = BOXES * V_TILE;
  static constexpr int STAGE_RAW = QK_BYTES + VPS * VB_BYTES;
  static constexpr int STAGE_BYTES = (STAGE_RAW + 1023) / 1024 * 1024;
  static_assert(!PAIRED || (QK_BYTES % 1024 == 0 && VB_BYTES % 1024 == 0), "1 KB aligned tiles");
  static constexpr int TX_QK = PARTS * (QROWS_PER_HEAD + KS) * ROWB;  // Q and K of every part
  // Q/K barrier groups per stage: paired, one per pair, so that the S and G
  // MMAs of heads 0-1 start once their pair has landed and the pair's next
  // load starts once those MMAs are done (the two pairs' loads and MMAs
  // pipeline at half-item granularity)
  static constexpr int QKG = PAIRED ? BOXES : 1;
  static constexpr int TX_QKG = TX_QK / QKG;
  static constexpr int BPG = BOXES / QKG;                 // boxes per group
  static constexpr int TX_V = PARTS * KP * ROWB;                       // V of every part
  static constexpr int P_TILE = WIN * 2048;               // 64 rows x 16 keys x 2 B per window row
  static constexpr int P_SMEM = PAIRED ? 0 : 2 * P_TILE;  // P tiles in shared memory (one per warpgroup)
  static constexpr int R_TILE = kGCols * ROWB;            // [rel_h; 0; rel_w; 0] B operand
  static constexpr int SCRATCH_LINE = 36;                 // floats per (row, half) line of the gather scratch
  static constexpr int SCRATCH = 8 * 32 * SCRATCH_LINE * 4;
  static constexpr bool SUM_BY_MMA = (D == 16);           // row sums through a ones tile in PV
  static constexpr int ONES_TILE = SUM_BY_MMA ? KP * ROWB : 0;
  static constexpr int O_COLS = SUM_BY_MMA ? 2 * D : D;   // PV N
  static constexpr SmemSwizzle SW = (ROWB == 32) ? SW_32B : (ROWB == 64 ? SW_64B : SW_128B);
  static constexpr uint32_t SBO = 8 * ROWB;               // 8-row core-matrix group stride
  static constexpr SmemSwizzle BSW = (BROWB == 32) ? SW_32B : (BROWB == 64 ? SW_64B : SW_128B);
  static constexpr uint32_t BSBO = 8 * BROWB;             // the same for the q/k/v tiles
  static constexpr int NROW = WIN / 2;                    // window rows per thread
  // Stride 2 with fewer than 4 parts: warpgroup 1's parts go to the upper
  // lane quadrants (its Q view starts QSHIFT rows earlier), so the two
  // warpgroups' active warps sit on different schedulers.
  static constexpr int QSHIFT = (STRIDE == 2 && PARTS <= 2) ? 32 : 0;
  // A.V issue streams: warp q < NST of the warpgroup issues a share of the
  // PARTS x WIN K-steps (part q / SPP, window rows of slice q % SPP) into its
  // own accumulator O_q at slot column q * O_COLS.
  static constexpr int NST = (O_COLS * 4 <= (int)kTmemG) ? 4 : 3;
  static constexpr int SPP = NST / PARTS;                 // streams per part
  static_assert(NST % PARTS == 0 && SPP >= 1, "streams per part");
  // Paired heads: the two pair tiles of V sit V_TILE apart, so one chain with
  // B = [V_0 V_1 | V_2 V_3] (N = 4d, each pair tile one 64-column N atom, at
  // leading byte offset V_TILE) replaces the four per-head chains; rows of
  // head p keep only columns p*d..p*d+d-1, which is where stream p's
  // accumulator was.  One issuer, a quarter of the MMAs.
  static constexpr bool AV_ONE_CHAIN = PAIRED;
  static_assert(!PAIRED || (SPP == 1 && !SUM_BY_MMA), "paired heads: one stream per head");
  static constexpr int NIS = AV_ONE_CHAIN ? 1 : NST;      // A.V issuers (commits per item)
  // the one chain is issued by warp 11 (otherwise idle), not by a softmax
  // warp, which would stall on a full MMA queue instead of moving on
  static constexpr bool AV_WARP = AV_ONE_CHAIN;
  // first O column of a slot: paired, P (8 columns per window row) sits at
  // [0, 8w) and O at [128, 256), over S's tail and G, both read by then
  static constexpr int O_BASE = PAIRED ? 128 : 0;
  static_assert(!PAIRED || (8 * WIN <= O_BASE && O_BASE + PARTS * D <= (int)kSlotCols), "paired TMEM slot");
  static_assert(NST * O_COLS <= (int)kTmemG, "O accumulators below the G columns");
  static_assert(WIN % 2 == 0 && WIN <= 14 && WIN >= 8, "window must be even, 8..14");
  static_assert(D == 16 || D == 32 || D == 64, "dim_head must be 16, 32 or 64");
  static_assert(NS <= (int)kTmemG, "S must fit below G in a TMEM slot");
  static_assert(2 * WIN - 1 <= kGRelW, "relative table rows");
};

// Bytes of dynamic shared memory for a given stage count (plus 1 KB alignment slack).
template <int D, int WIN, int STRIDE, int PP>
__host__ __device__ constexpr int smem_bytes(int stages) {
  using C = Cfg<D, WIN, STRIDE, PP>;
  return 1024 + C::P_SMEM + C::SCRATCH + ((C::R_TILE + 1023) / 1024) * 1024 + stages * C::STAGE_BYTES +
         C::ONES_TILE;
}

// Swizzled byte offset of 16-byte unit u of row r in a K-major tile whose
// rows are ROWB bytes (the TMA / tcgen05 32B, 64B and 128B swizzle patterns).
template <int ROWB>
__device__ __forceinline__ uint32_t swz(int r, int u) {
  if (ROWB == 32) return r * 32 + ((u ^ ((r >> 2) & 1)) << 4);
  if (ROWB == 64) return r * 64 + ((u ^ ((r >> 1) & 3)) << 4);
  return r * 128 + ((u ^ (r & 7)) << 4);
}

__device__ __forceinline__ float exp2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void record_timeout(int* abort_flag) {
  atomicExch(&g_halo_error, -8);  // HALO_ERR_TIMEOUT
  *(volatile int*)abort_flag = 1;
}

struct ItemCoord {
  int n, by, bx, grp;
};

__device__ __forceinline__ ItemCoord item_coord(int item, int groups, int nbx, int nby) {
  ItemCoord c;
  c.grp = item % groups;
  const int blk = item / groups;
  c.bx = blk % nbx;
  c.by = (blk / nbx) % nby;
  c.n = blk / (nbx * nby);
  return c;
}

template <int D, int WIN, int STRIDE, int PP>
__global__ void __launch_bounds__(kThreads, 1)
    halo_fwd_tc(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                const __grid_constant__ CUtensorMap tmap_v, const Params p) {
  using C = Cfg<D, WIN, STRIDE, PP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sP = smem;                                          // P tiles (one per warpgroup) unless in TMEM
  float* sScratch = reinterpret_cast<float*>(sP + C::P_SMEM);  // relative-logit gather scratch
  uint8_t* sR = sP + C::P_SMEM + C::SCRATCH;                   // R tile (1 KB aligned)
  uint8_t* sStage = sR + ((C::R_TILE + 1023) / 1024) * 1024;   // stages x STAGE_BYTES
  // ones tile (d = 16) after the stages: the PV B descriptor reaches it with a
  // positive leading byte offset from any V tile
  uint8_t* sOnes = sStage + p.stages * C::STAGE_BYTES;

  // Q/K and V of a stage have their own barriers: Q and K are released when
  // the S and G MMAs finish, long before the A.V releases V, so the next
  // items' Q/K loads are in flight during the softmax.
  __shared__ __align__(8) uint64_t bar_fqk[16];  // index QKG * stage + group
  // V of item k lands on bar_fv[k % (2 SVB)]: a barrier per V buffer and per
  // warpgroup, so that the A.V issuer of item k never waits on a barrier
  // whose previous phase (the other warpgroup's item k - 1, with one buffer)
  // is still open, where a parity wait would pass one phase early.
  __shared__ __align__(8) uint64_t bar_fv[16];
  __shared__ __align__(8) uint64_t bar_eqk[16];  // count 2: the S and the G MMAs of the group
  __shared__ __align__(8) uint64_t bar_ev[8];   // V buffer free; count NIS: the A.V issuers
  __shared__ __align__(8) uint64_t bar_sfull[4];   // index 2*g + slot
  __shared__ __align__(8) uint64_t bar_pfull[4];
  __shared__ __align__(8) uint64_t bar_ofull[4];
  __shared__ __align__(8) uint64_t bar_tfree[4];
  __shared__ __align__(8) uint64_t bar_done[3];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int S = p.stages;
  const int SVB = C::VPS * S;  // V buffers: item k's V in buffer k % SVB
  auto vbuf = [&](int k) -> uint8_t* {
    const int vb = k % SVB;
    return sStage + (vb / C::VPS) * C::STAGE_BYTES + C::QK_BYTES + (vb % C::VPS) * C::VB_BYTES;
  };

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      for (int q = 0; q < C::QKG; ++q) {
        mbar_init(&bar_fqk[C::QKG * i + q], 1);
        mbar_init(&bar_eqk[C::QKG * i + q], 2);
      }
    }
    for (int i = 0; i < SVB; ++i) {
      mbar_init(&bar_fv[i], 1);
      mbar_init(&bar_fv[SVB + i], 1);
      mbar_init(&bar_ev[i], C::NIS);
    }
    for (int b = 0; b < 4; ++b) {
      mbar_init(&bar_sfull[b], 2);  // the S MMAs (warp 9) and the G MMAs (warp 10)
      mbar_init(&bar_pfull[b], 4);
      mbar_init(&bar_ofull[b], C::NIS);
      mbar_init(&bar_tfree[b], 4);
    }
    mbar_init(&bar_done[0], 1);
    mbar_init(&bar_done[1], 1);
    mbar_init(&bar_done[2], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kTmaWarp && lane == 0) {
    prefetch_tensormap(&tmap_q);
    prefetch_tensormap(&tmap_k);
    prefetch_tensormap(&tmap_v);
  }
  // R tile: rows [0, 2w-1) = rel_h, rows [28, 28+2w-1) = rel_w, other rows 0.
  for (int idx = tid; idx < kGCols * (D / 8); idx += kThreads) {
    const int r = idx / (D / 8), u = idx % (D / 8);
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r < 2 * WIN - 1) val = *reinterpret_cast<const uint4*>(p.rel_h + r * D + u * 8);
    else if (r >= kGRelW && r < kGRelW + 2 * WIN - 1)
      val = *reinterpret_cast<const uint4*>(p.rel_w + (r - kGRelW) * D + u * 8);
    *reinterpret_cast<uint4*>(sR + swz<C::ROWB>(r, u)) = val;
  }
  if constexpr (C::SUM_BY_MMA) {
    // ones tile in the same MN-major layout as a V tile: every element 1.0
    for (int idx = tid; idx < C::ONES_TILE / 16; idx += kThreads)
      reinterpret_cast<uint4*>(sOnes)[idx] = make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);
  }
  // Zero what the TMA never writes: the K tile rows KS..NS-1 (read by the
  // N = NS MMA) and, at stride 2, the query buffer outside the head slots.
  for (int s = 0; s < S; ++s) {
    uint8_t* st = sStage + s * C::STAGE_BYTES;
    if constexpr (STRIDE == 2) {
      for (int idx = tid; idx < C::Q_BYTES / 16; idx += kThreads)
        reinterpret_cast<uint4*>(st)[idx] = make_uint4(0, 0, 0, 0);
    }
    if constexpr (C::NS > C::KS) {
      constexpr int tail = (C::NS - C::KS) * C::BROWB / 16;
      for (int idx = tid; idx < C::BOXES * tail; idx += kThreads) {
        uint8_t* kt = st + C::Q_BYTES + (idx / tail) * C::K_TILE + C::KS * C::BROWB;
        reinterpret_cast<uint4*>(kt)[idx % tail] = make_uint4(0, 0, 0, 0);
      }
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

  // Items of this CTA: k = 0, 1, ...; global item = blockIdx.x + k * gridDim.x
  // ordered so that concurrently running CTAs work on neighbouring blocks.
  // Item k belongs to warpgroup k & 1 as its (k >> 1)-th item, which uses
  // TMEM slot (k >> 1) & 1 of that warpgroup.
  const int groups = p.heads / C::PARTS;
  const int my_items = (p.num_items > (int)blockIdx.x)
                           ? (p.num_items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (warp >= 8) {
  // Producer warpgroup.  Each role ends in its own copy of the teardown
  // barrier so that no code is shared between the two register budgets.
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    // issue order QK(0), QK(1), V(0), QK(2), V(1), ...: the Q/K of an item
    // go out one item ahead of the V it does not need until its A.V
    if (lane == 0) {
      int nv = 0, nqkg = 0;  // items with V loads, groups with Q/K loads issued
      for (int t = 0; t <= my_items; ++t) {
        if (t < my_items) {
          const int s = t % S;
          const ItemCoord ic = item_coord(blockIdx.x + t * gridDim.x, groups, p.nbx, p.nby);
          uint8_t* st = sStage + s * C::STAGE_BYTES;
          bool waited = true;
#pragma unroll 1
          for (int q = 0; q < C::QKG && waited; ++q) {
            uint64_t* fqk = &bar_fqk[C::QKG * s + q];
            waited = t < S || mbar_wait(&bar_eqk[C::QKG * s + q], ((t / S) - 1) & 1, kWaitNs, &abort_flag);
            if (!waited) break;
            mbar_arrive_expect_tx(fqk, C::TX_QKG);
#pragma unroll 1
            for (int box = q * C::BPG; box < (q + 1) * C::BPG; ++box) {
              const int head = ic.grp * C::PARTS + box * C::HPB;
              uint8_t* qdst = st + ((STRIDE == 1) ? 0 : C::q_row(box) * C::BROWB);
              tma_load_4d(qdst, &tmap_q, fqk, head * D, ic.bx * kBlock, ic.by * kBlock, ic.n);
              uint8_t* kdst = st + C::Q_BYTES + box * C::K_TILE;
              tma_load_4d(kdst, &tmap_k, fqk, head * D, ic.bx * kBlock - p.halo, ic.by * kBlock - p.halo, ic.n);
            }
            nqkg = C::QKG * t + q + 1;
          }
          if (!waited) {
            if (!abort_flag) record_timeout(&abort_flag);
            break;
          }
        }
        if (t >= 1) {
          const int k = t - 1, vb = k % SVB;
          if (k >= SVB && !mbar_wait(&bar_ev[vb], ((k / SVB) - 1) & 1, kWaitNs, &abort_flag)) {
            if (!abort_flag) record_timeout(&abort_flag);
            break;
          }
          const ItemCoord ic = item_coord(blockIdx.x + k * gridDim.x, groups, p.nbx, p.nby);
          uint8_t* vt = vbuf(k);
          uint64_t* fv = &bar_fv[k % (2 * SVB)];
          mbar_arrive_expect_tx(fv, C::TX_V);
#pragma unroll 1
          for (int box = 0; box < C::BOXES; ++box) {
            const int head = ic.grp * C::PARTS + box * C::HPB;
            uint8_t* vdst = vt + box * C::V_TILE;
            tma_load_4d(vdst, &tmap_v, fv, head * D, ic.bx * kBlock - p.halo, ic.by * kBlock - p.halo,
                        ic.n);
          }
          nv = k + 1;
        }
      }
      if (abort_flag) {
        // let loads that are still in flight land before the CTA exits
        for (int u = (nqkg > C::QKG * S ? nqkg - C::QKG * S : 0); u < nqkg; ++u) {
          const int k = u / C::QKG, q = u % C::QKG;
          mbar_wait(&bar_fqk[C::QKG * (k % S) + q], (k / S) & 1, kWaitNs);
        }
        for (int k = (nv > SVB ? nv - SVB : 0); k < nv; ++k)
          mbar_wait(&bar_fv[k % (2 * SVB)], (k / (2 * SVB)) & 1, kWaitNs);
      }
    }
  } else if (warp == kMmaWarp || warp == kMmaWarp + 1) {
    // warp 9 issues S = Q K^T, warp 10 G = Q R^T, in parallel
    const bool is_g = (warp == kMmaWarp + 1);
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(64, C::NS, false);
      const uint32_t idG = idesc_bf16_f32(64, kGCols, false);
      // S(k): QK^T and the relative dot products of item k into its TMEM slot.
      // Group q: the heads of its boxes; the last group commits sfull.
      auto issue_s = [&](int k, int q) {
        const int s = k % S, g = k & 1, sl = (k >> 1) & 1;
        const uint32_t dst = tmem + (static_cast<uint32_t>(g * 16) << 16) + sl * kSlotCols;
        const uint8_t* st = sStage + s * C::STAGE_BYTES;
        constexpr int PPG = C::PARTS / C::QKG;  // heads per group
        if (!is_g) {
#pragma unroll 1
          for (int part = q * PPG; part < (q + 1) * PPG; ++part) {
            const uint32_t qa =
                smem_addr(st + ((STRIDE == 1) ? 0 : (C::view_row(part) - g * C::QSHIFT) * C::BROWB) + C::koff(part));
            const uint32_t ka = smem_addr(st + C::Q_BYTES + (part / C::HPB) * C::K_TILE + C::koff(part));
            for (int ks = 0; ks < D / 16; ++ks) {
              mma_f16_ss(dst, smem_desc(qa + 32 * ks, 16, C::BSBO, C::BSW),
                         smem_desc(ka + 32 * ks, 16, C::BSBO, C::BSW), idS, (part | ks) != 0);
            }
          }
          if (q == C::QKG - 1) mma_commit(&bar_sfull[2 * g + sl]);
          mma_commit(&bar_eqk[C::QKG * s + q]);
          return;
        }
        const uint32_t ra = smem_addr(sR);
#pragma unroll 1
        for (int part = q * PPG; part < (q + 1) * PPG; ++part) {
          const uint32_t qa =
              smem_addr(st + ((STRIDE == 1) ? 0 : (C::view_row(part) - g * C::QSHIFT) * C::BROWB) + C::koff(part));
          for (int ks = 0; ks < D / 16; ++ks) {
            mma_f16_ss(dst + kTmemG, smem_desc(qa + 32 * ks, 16, C::BSBO, C::BSW),
                       smem_desc(ra + 32 * ks, 16, C::SBO, C::SW), idG, (part | ks) != 0);
          }
        }
        if (q == C::QKG - 1) mma_commit(&bar_sfull[2 * g + sl]);
        mma_commit(&bar_eqk[C::QKG * s + q]);
      };
      // S(k) needs its stage loaded and the slot's previous item (k - 4)
      // consumed (the A.V MMAs are issued by the softmax warpgroups)
      bool fine = true;
      for (int ns = 0; ns < my_items && fine; ++ns) {
        fine = ns < 4 || mbar_wait(&bar_tfree[2 * (ns & 1) + ((ns >> 1) & 1)], ((ns >> 2) - 1) & 1, kWaitNs,
                                   &abort_flag);
#pragma unroll 1
        for (int q = 0; q < C::QKG && fine; ++q) {
          fine = mbar_wait(&bar_fqk[C::QKG * (ns % S) + q], (ns / S) & 1, kWaitNs, &abort_flag);
          if (fine) {
            tc_fence_after();
            issue_s(ns, q);
          }
        }
      }
      if (!fine && !abort_flag) record_timeout(&abort_flag);
      // all issued MMAs complete before the CTA frees TMEM
      mma_commit(&bar_done[is_g ? 1 : 0]);
      mbar_wait(&bar_done[is_g ? 1 : 0], 0, kWaitNs);
    }
  } else if (C::AV_WARP && warp == kMmaWarp + 2) {
    // ------------------------------------------------------------ A.V issue (warp 11)
    // item k: once its warpgroup has stored P (pfull) and its V has landed,
    // O = P V as one chain over both pair tiles into the slot's O columns
    if (lane == 0) {
      const uint32_t idO = idesc_bf16_f32(64, C::PARTS * D, true);
      for (int k = 0; k < my_items; ++k) {
        const int g = k & 1, jj = k >> 1, sl = jj & 1, b = 2 * g + sl;
        if (!mbar_wait(&bar_pfull[b], (jj >> 1) & 1, kWaitNs, &abort_flag) ||
            !mbar_wait(&bar_fv[k % (2 * SVB)], (k / (2 * SVB)) & 1, kWaitNs, &abort_flag)) {
          if (!abort_flag) record_timeout(&abort_flag);
          break;
        }
        tc_fence_after();
        const uint32_t slot = tmem + (static_cast<uint32_t>(g * 16) << 16) + sl * kSlotCols;
        const uint32_t va = smem_addr(vbuf(k));
#pragma unroll 1
        for (int kk = 0; kk < WIN; ++kk)
          mma_f16_ts(slot + C::O_BASE, slot + 8 * kk,
                     smem_desc(va + kk * kRowKeys * C::BROWB, C::V_TILE, C::BSBO, C::BSW), idO, kk != 0);
        mma_commit(&bar_ofull[b]);
        mma_commit(&bar_ev[k % SVB]);
      }
      mma_commit(&bar_done[2]);
      mbar_wait(&bar_done[2], 0, kWaitNs);
    }
  }
  __syncwarp();  // reconverge lane 0 with its warp before the aligned barrier
  tc_fence_before();
  named_bar_sync(1, kThreads);
  return;
  }

  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
  {
    // ------------------------------------------------------------ softmax warpgroups
    const int g = warp >> 2;          // warpgroup 0 or 1
    const int wq = warp & 3;          // TMEM lane quadrant
    const int half = lane >> 4;       // 0: even window rows, 1: odd window rows
    const int r16 = lane & 15;        // row within the quadrant
    const int part_w = wq - g * (C::QSHIFT / 16);   // this warp's head part at stride 2
    const bool active = (STRIDE == 1) || (part_w >= 0 && part_w < C::PARTS);
    const uint32_t tq = tmem + (static_cast<uint32_t>(32 * wq + 16 * g) << 16);
    uint8_t* pt = sP + g * C::P_TILE;
    float* scr = sScratch + (warp * 32) * C::SCRATCH_LINE;  // this warp's 32 lines
    // this thread's query row within the 64-row tile, and its in-block offset
    const int row = 16 * wq + r16;
    const int qy = (STRIDE == 1) ? (row >> 3) : 2 * (r16 >> 2);
    const int qx = (STRIDE == 1) ? (row & 7) : 2 * (r16 & 3);
    const float c = p.c;
    const int C_all = p.heads * D;
    const uint32_t idO = idesc_bf16_f32(64, C::AV_ONE_CHAIN ? C::PARTS * D : C::O_COLS, true);

    // Epilogue of a finished item: O (and row sums) from its TMEM slot,
    // normalise, bf16, store; then hand the slot back to the MMA warp.
    auto epilogue = [&](int jj, const ItemCoord& ic, float l) -> bool {
      const int b = 2 * g + (jj & 1);
      if (!mbar_wait(&bar_ofull[b], (jj >> 1) & 1, kWaitNs, &abort_flag)) {
        if (!abort_flag) record_timeout(&abort_flag);
        return false;
      }
      tc_fence_after();
      // the streams of this warp's part: all of them at stride 1, part wq at stride 2
      float o[D / 2];
#pragma unroll
      for (int t = 0; t < D / 2; ++t) o[t] = 0.f;
      if (active) {
        const int q0 = (STRIDE == 1) ? 0 : part_w * C::SPP;
        if constexpr (D == 16) l = 0.f;
#pragma unroll 1
        for (int q = q0; q < q0 + ((STRIDE == 1) ? C::NST : C::SPP); ++q) {
          const uint32_t oaddr = tq + (jj & 1) * kSlotCols + C::O_BASE + q * C::O_COLS;
          if constexpr (D == 16) {
            uint32_t r[8];
            tmem_ld_16x32bx2_x8<8>(oaddr, r);
            uint32_t rs[8];
            tmem_ld_16x32bx2_x8<8>(oaddr + D, rs);  // row sums (ones tile): every column holds the sum
            tmem_wait_ld();
#pragma unroll
            for (int t = 0; t < 8; ++t) o[t] += __uint_as_float(r[t]);
            l += __uint_as_float(rs[0]);
          } else if constexpr (D == 32) {
            uint32_t r[16];
            tmem_ld_16x32bx2_x16<16>(oaddr, r);
            tmem_wait_ld();
#pragma unroll
            for (int t = 0; t < 16; ++t) o[t] += __uint_as_float(r[t]);
          } else {
            // two loads of 16 columns per half row: fewer registers live next
            // to the S rows of the item in flight
#pragma unroll
            for (int hpart = 0; hpart < 2; ++hpart) {
              uint32_t r[16];
              tmem_ld_16x32bx2_x16<32>(oaddr + 16 * hpart, r);
              tmem_wait_ld();
#pragma unroll
              for (int t = 0; t < 16; ++t) o[16 * hpart + t] += __uint_as_float(r[t]);
            }
          }
        }
      }
      // the slot's TMEM has been read: hand it back before the arithmetic and stores
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_tfree[b]);
      if (active) {
        const int head = ic.grp * C::PARTS + ((STRIDE == 1) ? 0 : part_w);
        const float inv = 1.0f / l;
        uint32_t pk[D / 4];
#pragma unroll
        for (int t = 0; t < D / 4; ++t) pk[t] = pack_bf16x2(o[2 * t] * inv, o[2 * t + 1] * inv);
        const int y = ic.by * kBlock + qy, x = ic.bx * kBlock + qx;
        const int oy = y / STRIDE, ox = x / STRIDE;
        __nv_bfloat16* dst =
            p.out + ((static_cast<size_t>(ic.n) * p.OH + oy) * p.OW + ox) * C_all + head * D + half * (D / 2);
#pragma unroll
        for (int t = 0; t < D / 16; ++t)
          reinterpret_cast<uint4*>(dst)[t] = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
      }
      return true;
    };

    ItemCoord prev_ic{0, 0, 0, 0};
    float prev_l = 0.f;
    int j = 0;
    bool ok = true;
    for (int k = g; k < my_items; k += 2, ++j) {
      const int sl = j & 1;
      const int b = 2 * g + sl;
      if (!mbar_wait(&bar_sfull[b], (j >> 1) & 1, kWaitNs, &abort_flag)) {
        if (!abort_flag) record_timeout(&abort_flag);
        ok = false;
        break;
      }
      tc_fence_after();
      const ItemCoord ic = item_coord(blockIdx.x + k * gridDim.x, groups, p.nbx, p.nby);
      const int y0 = ic.by * kBlock - p.halo, x0 = ic.bx * kBlock - p.halo;
      const uint32_t ts = tq + sl * kSlotCols;

      float rh[C::NROW];
      float rw[WIN];
      float sv[C::NROW][16];
      float m = -INFINITY;
      if (active) {
        // ---- relative logits: this query's G row -> scratch line -> gather
        {
          uint32_t gr[32];
          tmem_ld_16x32bx2_x32<24>(ts + kTmemG, gr);  // half 0: rel_h part, half 1: rel_w part (from col 24)
          tmem_wait_ld();
          float* line = scr + (2 * r16 + half) * C::SCRATCH_LINE;
#pragma unroll
          for (int t = 0; t < 8; ++t)
            reinterpret_cast<uint4*>(line)[t] =
                make_uint4(gr[4 * t + 0], gr[4 * t + 1], gr[4 * t + 2], gr[4 * t + 3]);
        }
        __syncwarp();
        const float* lh = scr + (2 * r16) * C::SCRATCH_LINE;                        // rel_h logits
        const float* lw = scr + (2 * r16 + 1) * C::SCRATCH_LINE + (kGRelW - 24);   // rel_w logits
#pragma unroll
        for (int i = 0; i < C::NROW; ++i) {
          const int kr = 2 * i + half;
          const int Y = y0 + kr;
          rh[i] = (Y >= 0 && Y < p.H) ? lh[kr - qy + WIN - 1] : -INFINITY;
        }
#pragma unroll
        for (int kc = 0; kc < WIN; ++kc) {
          const int X = x0 + kc;
          rw[kc] = (X >= 0 && X < p.W) ? lw[kc - qx + WIN - 1] : -INFINITY;
        }

        // ---- S rows of this thread: window rows 2i + half (WIN keys each)
#pragma unroll
        for (int i = 0; i < C::NROW; ++i)
          tmem_ld_16x32bx2_x16<WIN>(ts + 2 * WIN * i, *reinterpret_cast<uint32_t(*)[16]>(&sv[i][0]));
        tmem_wait_ld();

        // ---- exact row max of z = S + rel_h + rel_w over in-image keys
#pragma unroll
        for (int i = 0; i < C::NROW; ++i) {
          float mi = -INFINITY;
#pragma unroll
          for (int kc = 0; kc < WIN; ++kc) {
            sv[i][kc] += rw[kc];
            mi = fmaxf(mi, sv[i][kc]);
          }
          m = fmaxf(m, mi + rh[i]);
        }
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
      }
      tc_fence_before();

      // ---- finish the previous item while this one's P is not yet written:
      // its PV has had the whole gather + max to complete, and P(j-1) must be
      // consumed before P(j) overwrites the warpgroup's P tile.
      if (j >= 1 && !epilogue(j - 1, prev_ic, prev_l)) {
        ok = false;
        break;
      }

      float l = 0.f;
      if (active) {
        const float mc = m * c;
        // ---- p = 2^(c*z - c*m); bf16 P into the swizzled operand tile
#pragma unroll
        for (int i = 0; i < C::NROW; ++i) {
          const float bias = fmaf(rh[i], c, -mc);
          float e[16];
#pragma unroll
          for (int kc = 0; kc < 16; ++kc) {
            if (kc < WIN) {
              const float x = fmaf(sv[i][kc], c, bias);
              // every exponential on MUFU: here the unit runs at about 14% of
              // its rate, and moving 40% of them to the FMA-pipe polynomial
              // cost more issue slots than it saved (stride-2 workload 213.7
              // against 176.4 us)
              e[kc] = exp2_mufu(x);
            } else {
              e[kc] = 0.f;
            }
          }
          uint32_t pk[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) pk[t] = pack_bf16x2(e[2 * t], e[2 * t + 1]);
          if constexpr (!C::SUM_BY_MMA) {
#pragma unroll
            for (int kc = 0; kc < WIN; ++kc) l += e[kc];
          }
          if constexpr (C::PAIRED) {
            // window rows 2i (this lane < 16) and 2i + 1 (its partner) at
            // columns 16i and 16i + 8: 8 columns of bf16 pairs per K-step
            tmem_st_16x32bx2_x8<8>(ts + 16 * i, pk);
          } else {
            const int kr = 2 * i + half;
            uint8_t* dst = pt + kr * 2048 + row * 32;
            const int sw = (row >> 2) & 1;
            *reinterpret_cast<uint4*>(dst + (sw << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            *reinterpret_cast<uint4*>(dst + ((sw ^ 1) << 4)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
        if constexpr (!C::SUM_BY_MMA) l += __shfl_xor_sync(0xffffffffu, l, 16);
        if constexpr (C::PAIRED) {
          tmem_wait_st();
          tc_fence_before();
        } else {
          fence_proxy_async_smem();
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_pfull[b]);
      // ---- A.V: warp wq < NIS issues its share once the whole P tile is
      // written (with AV_WARP, warp 11 does)
      bool issued = true;
      if (!C::AV_WARP && wq < C::NIS && lane == 0) {
        issued = mbar_wait(&bar_pfull[b], (j >> 1) & 1, kWaitNs, &abort_flag) &&
                 mbar_wait(&bar_fv[k % (2 * SVB)], (k / (2 * SVB)) & 1, kWaitNs, &abort_flag);
        if (issued) {
          tc_fence_after();
          const int part = wq / C::SPP, sub = wq % C::SPP;
          const int kb = WIN * sub / C::SPP, ke = WIN * (sub + 1) / C::SPP;
          const uint32_t slot = tmem + (static_cast<uint32_t>(g * 16) << 16) + sl * kSlotCols;
          const uint32_t dst = slot + C::O_BASE + wq * C::O_COLS;
          const uint32_t va = smem_addr(vbuf(k) + part * C::V_TILE);
          // with the ones tile the B operand spans two swizzle atoms along N:
          // V (D columns) then ones (D columns) at leading byte offset LBO
          const uint32_t lbo = C::SUM_BY_MMA ? (smem_addr(sOnes) - va) : (C::AV_ONE_CHAIN ? C::V_TILE : 16u);
          if constexpr (C::PAIRED) {
#pragma unroll 1
            for (int kk = kb; kk < ke; ++kk)
              mma_f16_ts(dst, slot + 8 * kk, smem_desc(va + kk * kRowKeys * C::BROWB, lbo, C::BSBO, C::BSW), idO,
                         kk != kb);
          } else {
            const uint32_t pa = smem_addr(pt);
#pragma unroll 1
            for (int kk = kb; kk < ke; ++kk)
              mma_f16_ss(dst, smem_desc(pa + kk * 2048, 16, 256, SW_32B),
                         smem_desc(va + kk * kRowKeys * C::BROWB, lbo, C::BSBO, C::BSW), idO, kk != kb);
          }
          mma_commit(&bar_ofull[b]);
          mma_commit(&bar_ev[k % SVB]);
        }
      }
      if (!__all_sync(0xffffffffu, issued)) {
        if (!abort_flag) record_timeout(&abort_flag);
        ok = false;
        break;
      }
      prev_ic = ic;
      prev_l = l;
    }
    if (ok && j >= 1) epilogue(j - 1, prev_ic, prev_l);
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  named_bar_sync(1, kThreads);
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace tc
}  // namespace halo
