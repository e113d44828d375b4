// halo_api.cu -- host side of libhalo: argument checks, kernel selection,
// TMA descriptor encoding, launches, error reporting.  See include/halo.h for
// the contract of every entry point.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/halo.h"
#include "halo_bwd.cuh"
#include "halo_bwd_tc.cuh"
#include "halo_fused.cuh"
#include "halo_simt.cuh"
#include "halo_tc.cuh"
#include "halo_tc2.cuh"
#include "halo_tc3.cuh"
#include "halo_tc4.cuh"
#include "halo_win.cuh"

namespace {

constexpr int kVersion = 100;                 // 0.1.0
constexpr int kMaxDynSmem = 227 * 1024;       // sm_100 opt-in limit per block

const char* status_text(int code) {
  switch (code) {
    case HALO_OK: return "ok";
    case HALO_ERR_NULL: return "a required pointer is NULL";
    case HALO_ERR_DIMS: return "a size is non-positive or too large";
    case HALO_ERR_DIVISIBILITY: return "H and W must be multiples of block, and block a multiple of stride";
    case HALO_ERR_STRIDE: return "stride must be 1 or 2";
    case HALO_ERR_ALIGN: return "pointers must be 16-byte aligned and heads*dim_head rows a multiple of 16 bytes";
    case HALO_ERR_UNSUPPORTED: return "no kernel of this library handles this shape";
    case HALO_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case HALO_ERR_TIMEOUT: return "a bounded device-side wait ran out";
    case HALO_ERR_DTYPE: return "dtype must be HALO_F32 or HALO_BF16";
    case HALO_ERR_ALIAS: return "out overlaps an input";
    case HALO_ERR_DEVICE: return "the current device is not an sm_100 GPU";
    case HALO_ERR_KERNEL: return "the SASA mask size must be odd, and at most 2*halo+1";
    case HALO_ERR_WORKSPACE: return "the workspace is missing, misaligned or too small";
    case HALO_ERR_SCRATCH_LIMIT:
      return "the shape needs more scratch than halo_attn_bwd_noalloc's built-in 16 MiB (use halo_attn_bwd)";
    default: return "unknown status code";
  }
}

struct Shape {
  int N, H, W, heads, d, block, halo, stride, dtype;
  int kmask = 0;  // SASA mask size: 0 = none, else odd k with k / 2 <= halo
  size_t elem() const { return dtype == HALO_F32 ? 4 : 2; }
  size_t in_bytes() const { return static_cast<size_t>(N) * H * W * heads * d * elem(); }
  size_t out_bytes() const { return static_cast<size_t>(N) * (H / stride) * (W / stride) * heads * d * elem(); }
  size_t rel_bytes() const { return static_cast<size_t>(2 * (block + 2 * halo) - 1) * d * elem(); }
};

// Checks that need no pointers.  Order: dtype, sizes, stride, divisibility, row alignment.
int check_shape(const Shape& s) {
  if (s.dtype != HALO_F32 && s.dtype != HALO_BF16) return HALO_ERR_DTYPE;
  if (s.N <= 0 || s.H <= 0 || s.W <= 0 || s.heads <= 0 || s.d <= 0 || s.block <= 0 || s.halo < 0)
    return HALO_ERR_DIMS;
  const long long C = static_cast<long long>(s.heads) * s.d;
  const long long elems = static_cast<long long>(s.N) * s.H * s.W * C;
  if (C > (1 << 20) || elems >= (1LL << 40) || s.block + 2 * s.halo > 4096 || s.H > (1 << 24) ||
      s.W > (1 << 24))
    return HALO_ERR_DIMS;
  if (s.stride != 1 && s.stride != 2) return HALO_ERR_STRIDE;
  if (s.H % s.block || s.W % s.block || s.block % s.stride) return HALO_ERR_DIVISIBILITY;
  if ((C * static_cast<long long>(s.elem())) % 16 != 0) return HALO_ERR_ALIGN;
  if (s.kmask < 0 || (s.kmask > 0 && (s.kmask % 2 == 0 || s.kmask / 2 > s.halo))) return HALO_ERR_KERNEL;
  return HALO_OK;
}

// ----------------------------------------------------------------------------
// Tensor-core kernel table: (d, window, stride) -> instantiation
// ----------------------------------------------------------------------------
using TcKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const halo::tc::Params);

struct TcEntry {
  int d, win, stride;
  TcKernel fn;
  int (*smem)(int);
  int stage_bytes;
  int parts;
  int hpb;  // heads per TMA box
};

template <int D, int WIN, int STRIDE, int PP>
int tc_smem(int stages) { return halo::tc::smem_bytes<D, WIN, STRIDE, PP>(stages); }

#define HALO_TC_ENTRY(D, WIN, S, PP)                                                             \
  TcEntry {                                                                                      \
    D, WIN, S, halo::tc::halo_fwd_tc<D, WIN, S, PP>, tc_smem<D, WIN, S, PP>,                     \
        halo::tc::Cfg<D, WIN, S, PP>::STAGE_BYTES, PP, halo::tc::Cfg<D, WIN, S, PP>::HPB         \
  }
#define HALO_TC_WINS(D, S, PP)                                                                  \
  HALO_TC_ENTRY(D, 8, S, PP), HALO_TC_ENTRY(D, 10, S, PP), HALO_TC_ENTRY(D, 12, S, PP),         \
      HALO_TC_ENTRY(D, 14, S, PP)

// Stride 2 packs several heads into the 64-row tile (16 queries each): four
// where the head count allows (every softmax thread then has a query row),
// else two at d = 32; the first matching entry is taken.
const TcEntry kTcTable[] = {
    HALO_TC_WINS(16, 1, 1), HALO_TC_WINS(32, 1, 1), HALO_TC_WINS(64, 1, 1), HALO_TC_WINS(16, 2, 4),
    HALO_TC_WINS(32, 2, 4), HALO_TC_WINS(32, 2, 2), HALO_TC_WINS(64, 2, 1),
};

// Stride-1 kernel with two heads per 128-row tile (maps with an odd number of
// block rows): (d, window) -> instantiation.
using Tc2Kernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const halo::tc2::Params);
struct Tc2Entry {
  int d, win;
  Tc2Kernel fn;
  int (*smem)(int);
};
template <int D, int WIN>
int tc2_smem(int stages) { return halo::tc2::smem_bytes<D, WIN>(stages); }
#define HALO_TC2_ENTRY(D, WIN) \
  Tc2Entry { D, WIN, halo::tc2::halo_fwd_tc2<D, WIN>, tc2_smem<D, WIN> }
const Tc2Entry kTc2Table[] = {
    HALO_TC2_ENTRY(16, 8),  HALO_TC2_ENTRY(16, 10), HALO_TC2_ENTRY(16, 12), HALO_TC2_ENTRY(16, 14),
    HALO_TC2_ENTRY(32, 8),  HALO_TC2_ENTRY(32, 10), HALO_TC2_ENTRY(32, 12), HALO_TC2_ENTRY(32, 14),
};

const Tc2Entry* find_tc2(const Shape& s) {
  if (s.dtype != HALO_BF16 || s.block != halo::tc2::kBlock || s.stride != 1 || s.heads % 2) return nullptr;
  const int win = s.block + 2 * s.halo;
  for (const Tc2Entry& e : kTc2Table)
    if (e.d == s.d && e.win == win) return &e;
  return nullptr;
}

// Stride-1 kernel for 16x16 query blocks: (d, window) -> instantiation.
using Tc3Kernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const halo::tc3::Params);
struct Tc3Entry {
  int d, win, block;
  Tc3Kernel fn;
  int (*smem)(int);
};
template <int D, int WIN, int BLOCK>
int tc3_smem(int stages) { return halo::tc3::smem_bytes<D, WIN, BLOCK>(stages); }
#define HALO_TC3_ENTRY(D, WIN, B) \
  Tc3Entry { D, WIN, B, halo::tc3::halo_fwd_tc3<D, WIN, B>, tc3_smem<D, WIN, B> }
#define HALO_TC3_WINS(D)                                                                                   \
  HALO_TC3_ENTRY(D, 16, 16), HALO_TC3_ENTRY(D, 18, 16), HALO_TC3_ENTRY(D, 20, 16), HALO_TC3_ENTRY(D, 22, 16), \
      HALO_TC3_ENTRY(D, 24, 16), HALO_TC3_ENTRY(D, 32, 32), HALO_TC3_ENTRY(D, 34, 32),                      \
      HALO_TC3_ENTRY(D, 36, 32), HALO_TC3_ENTRY(D, 38, 32)
const Tc3Entry kTc3Table[] = {HALO_TC3_WINS(16), HALO_TC3_WINS(32)};

// 16x16 blocks (halo <= 4) and 32x32 blocks (halo <= 3: global attention on
// a 32x32 map, and the block-32 detection setting)
const Tc3Entry* find_tc3(const Shape& s) {
  if (s.dtype != HALO_BF16 || (s.block != 16 && s.block != 32) || s.stride != 1) return nullptr;
  const int win = s.block + 2 * s.halo;
  for (const Tc3Entry& e : kTc3Table)
    if (e.d == s.d && e.win == win && e.block == s.block) return &e;
  return nullptr;
}

// Stride-1 kernel with two vertically adjacent blocks of one head per item
// (maps with an even number of block rows; taken before the head-pair kernel).
using Tc4Kernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const halo::tc4::Params);
struct Tc4Entry {
  int d, win;
  Tc4Kernel fn, fn_masked;  // fn_masked: the SASA-masked instantiation
  int (*smem)(int);
};
template <int D, int WIN>
int tc4_smem(int stages) { return halo::tc4::smem_bytes<D, WIN>(stages); }
#define HALO_TC4_ENTRY(D, WIN)                                                                     \
  Tc4Entry {                                                                                       \
    D, WIN, halo::tc4::halo_fwd_tc4<D, WIN, false>, halo::tc4::halo_fwd_tc4<D, WIN, true>,         \
        tc4_smem<D, WIN>                                                                           \
  }
const Tc4Entry kTc4Table[] = {
    HALO_TC4_ENTRY(16, 8), HALO_TC4_ENTRY(16, 10), HALO_TC4_ENTRY(16, 12), HALO_TC4_ENTRY(16, 14),
    HALO_TC4_ENTRY(32, 8), HALO_TC4_ENTRY(32, 10), HALO_TC4_ENTRY(32, 12), HALO_TC4_ENTRY(32, 14),
    HALO_TC4_ENTRY(64, 8), HALO_TC4_ENTRY(64, 10), HALO_TC4_ENTRY(64, 12), HALO_TC4_ENTRY(64, 14),
};

const Tc4Entry* find_tc4(const Shape& s) {
  if (s.dtype != HALO_BF16 || s.block != halo::tc4::kBlock || s.stride != 1 || (s.H / s.block) % 2) return nullptr;
  const int win = s.block + 2 * s.halo;
  for (const Tc4Entry& e : kTc4Table)
    if (e.d == s.d && e.win == win) return &e;
  return nullptr;
}

const TcEntry* find_tc(const Shape& s) {
  if (s.dtype != HALO_BF16 || s.block != halo::tc::kBlock) return nullptr;
  const int win = s.block + 2 * s.halo;
  for (const TcEntry& e : kTcTable)
    if (e.d == s.d && e.win == win && e.stride == s.stride && s.heads % e.parts == 0) return &e;
  return nullptr;
}

int select_kernel(const Shape& s) {
  if (check_shape(s) != HALO_OK) return HALO_KERNEL_NONE;
  if (s.kmask == 0 && (find_tc4(s) || find_tc2(s) || find_tc(s) || find_tc3(s))) return HALO_KERNEL_TC_BF16;
  if (s.kmask > 0 && find_tc4(s)) return HALO_KERNEL_TC_BF16;
  if (s.d <= 128) return HALO_KERNEL_SIMT_F32;
  return HALO_KERNEL_NONE;
}

// ----------------------------------------------------------------------------
// Device properties and TMA descriptor encoding
// ----------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_mutex;
EncodeTiledFn g_encode = nullptr;
constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices];
int g_dev_ok[kMaxDevices];  // 0 unknown, 1 sm_100, -1 other

int device_info(int* sm_count) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HALO_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_dev_ok[dev] == 0) {
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return HALO_ERR_CUDA;
    g_dev_ok[dev] = (major == 10) ? 1 : -1;
    g_sm_count[dev] = sms;
  }
  if (g_dev_ok[dev] != 1) return HALO_ERR_DEVICE;
  *sm_count = g_sm_count[dev];
  return HALO_OK;
}

EncodeTiledFn encoder() {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  return g_encode;
}

// 4-D map over an NHWC bf16 tensor {C, W, H, N}; box {hpb * d, bw, bh, 1}
// (hpb heads' channels per box row), swizzled by the box row's width.
bool encode_nhwc(CUtensorMap* m, const void* base, const Shape& s, int bw, int bh, int estride, int hpb = 1) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  const cuuint64_t C = static_cast<cuuint64_t>(s.heads) * s.d;
  cuuint64_t dims[4] = {C, static_cast<cuuint64_t>(s.W), static_cast<cuuint64_t>(s.H),
                        static_cast<cuuint64_t>(s.N)};
  cuuint64_t strides[3] = {C * 2, C * 2 * s.W, C * 2 * s.W * s.H};
  const int inner = s.d * hpb;
  cuuint32_t box[4] = {static_cast<cuuint32_t>(inner), static_cast<cuuint32_t>(bw), static_cast<cuuint32_t>(bh), 1};
  cuuint32_t es[4] = {1, static_cast<cuuint32_t>(estride), static_cast<cuuint32_t>(estride), 1};
  const CUtensorMapSwizzle sw = inner == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                                            : (inner == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

int check_pointers(const void* q, const void* k, const void* v, const void* rel_h, const void* rel_w,
                   const void* out, const Shape& s) {
  if (!q || !k || !v || !rel_h || !rel_w || !out) return HALO_ERR_NULL;
  const void* ptrs[6] = {q, k, v, rel_h, rel_w, out};
  for (const void* ptr : ptrs)
    if (reinterpret_cast<uintptr_t>(ptr) % 16) return HALO_ERR_ALIGN;
  const size_t ob = s.out_bytes(), ib = s.in_bytes(), rb = s.rel_bytes();
  if (overlaps(out, ob, q, ib) || overlaps(out, ob, k, ib) || overlaps(out, ob, v, ib) ||
      overlaps(out, ob, rel_h, rb) || overlaps(out, ob, rel_w, rb))
    return HALO_ERR_ALIAS;
  return HALO_OK;
}

template <typename T, int DMAX>
cudaError_t launch_simt_t(const void* q, const void* k, const void* v, const void* rh, const void* rw, void* out,
                          const Shape& s, cudaStream_t st) {
  const long long total = static_cast<long long>(s.N) * (s.H / s.stride) * (s.W / s.stride) * s.heads;
  const long long blocks = (32 * total + halo::simt::kThreads - 1) / halo::simt::kThreads;  // a warp each
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  halo::simt::halo_fwd_simt<T, DMAX><<<static_cast<unsigned>(blocks), halo::simt::kThreads, 0, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), static_cast<const T*>(rh),
      static_cast<const T*>(rw), static_cast<T*>(out), s.N, s.H, s.W, s.heads, s.d, s.block, s.halo, s.stride,
      s.kmask, 1.0f / std::sqrt(static_cast<float>(s.d)));
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_simt(const void* q, const void* k, const void* v, const void* rh, const void* rw, void* out,
                        const Shape& s, cudaStream_t st) {
  if (s.d <= 16) return launch_simt_t<T, 16>(q, k, v, rh, rw, out, s, st);
  if (s.d <= 32) return launch_simt_t<T, 32>(q, k, v, rh, rw, out, s, st);
  if (s.d <= 64) return launch_simt_t<T, 64>(q, k, v, rh, rw, out, s, st);
  return launch_simt_t<T, 128>(q, k, v, rh, rw, out, s, st);
}

// Window-staged CUDA-core kernel: dim_head 8, 16, 32, 64 or 128 and one
// block's window (k, v and the tables as float32) within shared memory.
bool win_plan(const Shape& s, halo::win::Params* p, int* threads, int* smem) {
  if (s.d != 8 && s.d != 16 && s.d != 32 && s.d != 64 && s.d != 128) return false;
  const int w = s.block + 2 * s.halo;
  if (w > 64) return false;
  const int tt = s.d >= 16 ? s.d / 16 : 1;
  p->N = s.N;
  p->H = s.H;
  p->W = s.W;
  p->heads = s.heads;
  p->block = s.block;
  p->halo = s.halo;
  p->stride = s.stride;
  p->kmask = s.kmask;
  p->w = w;
  p->nqx = s.block / s.stride;
  p->nq = p->nqx * p->nqx;
  p->nbx = s.W / s.block;
  p->nby = s.H / s.block;
  p->qpass = p->nq < halo::win::kMaxThreads / tt ? p->nq : halo::win::kMaxThreads / tt;
  p->c = 1.4426950408889634f / std::sqrt(static_cast<float>(s.d));
  *threads = (p->qpass * tt + 31) / 32 * 32;
  *smem = halo::win::smem_floats(s.d, w, p->qpass) * 4;
  return *smem <= kMaxDynSmem;
}

template <typename T, int D>
int launch_win_t(const void* q, const void* k, const void* v, const void* rh, const void* rw, void* out,
                 const Shape& s, const halo::win::Params& p, int threads, int smem, cudaStream_t st) {
  auto fn = halo::win::halo_fwd_win<T, D>;
  if (cudaFuncSetAttribute(reinterpret_cast<const void*>(fn), cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return HALO_ERR_CUDA;
  const long long items = static_cast<long long>(s.N) * p.nby * p.nbx * s.heads;
  if (items > 0x7fffffffLL) return HALO_ERR_DIMS;
  fn<<<static_cast<unsigned>(items), threads, smem, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), static_cast<const T*>(rh),
      static_cast<const T*>(rw), static_cast<T*>(out), p);
  return cudaGetLastError() == cudaSuccess ? HALO_OK : HALO_ERR_CUDA;
}

template <typename T>
int launch_win(const void* q, const void* k, const void* v, const void* rh, const void* rw, void* out,
               const Shape& s, const halo::win::Params& p, int threads, int smem, cudaStream_t st) {
  switch (s.d) {
    case 8: return launch_win_t<T, 8>(q, k, v, rh, rw, out, s, p, threads, smem, st);
    case 16: return launch_win_t<T, 16>(q, k, v, rh, rw, out, s, p, threads, smem, st);
    case 32: return launch_win_t<T, 32>(q, k, v, rh, rw, out, s, p, threads, smem, st);
    case 64: return launch_win_t<T, 64>(q, k, v, rh, rw, out, s, p, threads, smem, st);
    case 128: return launch_win_t<T, 128>(q, k, v, rh, rw, out, s, p, threads, smem, st);
    default: return HALO_ERR_UNSUPPORTED;
  }
}

// What every tensor-core kernel's launch shares: the register split check
// (the kernels move registers between warpgroups with setmaxnreg, which is
// only safe when the launch's allocation covers the split; otherwise the
// increase would wait forever, so the launch is refused), the number of
// pipeline stages that fit the opt-in shared memory next to the kernel's
// static shared memory, and a persistent grid of one CTA per SM.
// opt_bytes / opt_flag: shared memory a kernel can use for an optional
// feature; the flag is set (and the bytes added) only when they fit next to
// the stages chosen without them.
template <class Params>
int launch_persistent(void (*fn)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const Params),
                      int threads, int softmax_regs, int producer_regs, int (*smem_fn)(int), int max_stages,
                      const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, Params& p,
                      long long items, int sm_count, cudaStream_t st, int opt_bytes = 0,
                      int Params::*opt_flag = nullptr) {
  cudaFuncAttributes attr;
  if (cudaFuncGetAttributes(&attr, reinterpret_cast<const void*>(fn)) != cudaSuccess) return HALO_ERR_CUDA;
  if (256 * softmax_regs + 128 * producer_regs > threads * attr.numRegs) return HALO_ERR_UNSUPPORTED;
  int optin = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return HALO_ERR_CUDA;
  const int budget = (optin < kMaxDynSmem ? optin : kMaxDynSmem) - static_cast<int>(attr.sharedSizeBytes);
  int stages = max_stages;
  while (stages > 1 && smem_fn(stages) > budget) --stages;
  int smem = smem_fn(stages);
  if (smem > budget) return HALO_ERR_UNSUPPORTED;
  if (opt_flag) {
    p.*opt_flag = (opt_bytes > 0 && smem + opt_bytes <= budget) ? 1 : 0;
    if (p.*opt_flag) smem += opt_bytes;
  }
  if (cudaFuncSetAttribute(reinterpret_cast<const void*>(fn), cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return HALO_ERR_CUDA;
  if (items > 0x7fffffffLL) return HALO_ERR_DIMS;
  p.num_items = static_cast<int>(items);
  p.stages = stages;
  const int grid = static_cast<int>(items < sm_count ? items : sm_count);
  fn<<<grid, threads, smem, st>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? HALO_OK : HALO_ERR_CUDA;
}

// Fields every tensor-core kernel's Params has.
template <class Params>
void fill_common(Params& p, const void* rh, const void* rw, void* out, const Shape& s) {
  p.rel_h = static_cast<const __nv_bfloat16*>(rh);
  p.rel_w = static_cast<const __nv_bfloat16*>(rw);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.N = s.N;
  p.H = s.H;
  p.W = s.W;
  p.heads = s.heads;
  p.halo = s.halo;
  p.c = 1.4426950408889634f / std::sqrt(static_cast<float>(s.d));
}

int launch_tc(const TcEntry& e, const void* q, const void* k, const void* v, const void* rh, const void* rw,
              void* out, const Shape& s, int sm_count, cudaStream_t st) {
  const int win = s.block + 2 * s.halo;
  CUtensorMap mq, mk, mv;
  if (!encode_nhwc(&mq, q, s, halo::tc::kBlock, halo::tc::kBlock, s.stride, e.hpb) ||
      !encode_nhwc(&mk, k, s, win, win, 1, e.hpb) || !encode_nhwc(&mv, v, s, halo::tc::kRowKeys, win, 1, e.hpb))
    return HALO_ERR_CUDA;
  halo::tc::Params p;
  fill_common(p, rh, rw, out, s);
  p.nbx = s.W / halo::tc::kBlock;
  p.nby = s.H / halo::tc::kBlock;
  p.heads_per_item = e.parts;
  p.OH = s.H / s.stride;
  p.OW = s.W / s.stride;
  const long long items = static_cast<long long>(s.N) * p.nbx * p.nby * (s.heads / e.parts);
  // eight V-buffer barriers: paired heads have two V buffers per stage
  return launch_persistent(e.fn, halo::tc::kThreads, halo::tc::kSoftmaxRegs, halo::tc::kProducerRegs, e.smem,
                           e.hpb == 2 ? 4 : 8, mq, mk, mv, p, items, sm_count, st);
}

int launch_tc2(const Tc2Entry& e, const void* q, const void* k, const void* v, const void* rh, const void* rw,
               void* out, const Shape& s, int sm_count, cudaStream_t st) {
  const int win = s.block + 2 * s.halo;
  CUtensorMap mq, mk, mv;
  if (!encode_nhwc(&mq, q, s, halo::tc2::kBlock, halo::tc2::kBlock, 1) || !encode_nhwc(&mk, k, s, win, win, 1) ||
      !encode_nhwc(&mv, v, s, win, win, 1))
    return HALO_ERR_CUDA;
  halo::tc2::Params p;
  fill_common(p, rh, rw, out, s);
  p.nbx = s.W / halo::tc2::kBlock;
  p.nby = s.H / halo::tc2::kBlock;
  const long long items = static_cast<long long>(s.N) * p.nbx * p.nby * (s.heads / 2);
  return launch_persistent(e.fn, halo::tc2::kThreads, halo::tc2::kSoftmaxRegs, halo::tc2::kProducerRegs, e.smem, 8,
                           mq, mk, mv, p, items, sm_count, st);
}

int launch_tc3(const Tc3Entry& e, const void* q, const void* k, const void* v, const void* rh, const void* rw,
               void* out, const Shape& s, int sm_count, cudaStream_t st) {
  const int win = s.block + 2 * s.halo;
  CUtensorMap mq, mk, mv;
  // Q box: the item's 256 queries (a whole 16x16 block, or 8 rows of a 32x32
  // block); K / V box: window rows padded to the kernel's row pitch (block
  // 32: a multiple of 8)
  const int pitch = e.block == 16 ? win : (win + 7) / 8 * 8;
  if (!encode_nhwc(&mq, q, s, e.block, 256 / e.block, 1) || !encode_nhwc(&mk, k, s, pitch, win, 1) ||
      !encode_nhwc(&mv, v, s, pitch, win, 1))
    return HALO_ERR_CUDA;
  halo::tc3::Params p;
  fill_common(p, rh, rw, out, s);
  p.nbx = s.W / e.block;
  p.nby = s.H / e.block;
  // output map: box = one softmax warp's 32 query rows (block x 32/block)
  if (!encode_nhwc(&p.tmap_o, out, s, e.block, 32 / e.block, 1)) return HALO_ERR_CUDA;
  const int quarters = e.block * e.block / 256;
  const long long items = static_cast<long long>(s.N) * p.nbx * p.nby * s.heads * quarters;
  // the kernel has four stage barriers; the output staging (8 warps x 32
  // rows) is used where it fits next to the stages
  return launch_persistent(e.fn, halo::tc3::kThreads, halo::tc3::kSoftmaxRegs, halo::tc3::kProducerRegs, e.smem, 4,
                           mq, mk, mv, p, items, sm_count, st, 8 * 32 * s.d * 2, &halo::tc3::Params::tma_out);
}

int launch_tc4(const Tc4Entry& e, const void* q, const void* k, const void* v, const void* rh, const void* rw,
               void* out, const Shape& s, int sm_count, cudaStream_t st) {
  const int win = s.block + 2 * s.halo;
  CUtensorMap mq, mk, mv;
  if (!encode_nhwc(&mq, q, s, halo::tc4::kBlock, halo::tc4::kBlock, 1) ||
      !encode_nhwc(&mk, k, s, win, win + halo::tc4::kBlock, 1) ||
      !encode_nhwc(&mv, v, s, win, win + halo::tc4::kBlock, 1))
    return HALO_ERR_CUDA;
  halo::tc4::Params p;
  fill_common(p, rh, rw, out, s);
  p.nbx = s.W / halo::tc4::kBlock;
  p.npy = s.H / (2 * halo::tc4::kBlock);
  p.kmask = s.kmask;
  const long long items = static_cast<long long>(s.N) * p.nbx * p.npy * s.heads;
  // the kernel has four stage barriers
  return launch_persistent(s.kmask > 0 ? e.fn_masked : e.fn, halo::tc4::kThreads, halo::tc4::kSoftmaxRegs,
                           halo::tc4::kProducerRegs, e.smem, 4, mq, mk, mv, p, items, sm_count, st);
}

int attn_device(const void* q, const void* k, const void* v, const void* rel_h, const void* rel_w, void* out,
                const Shape& s, cudaStream_t st) {
  int rc = check_shape(s);
  if (rc != HALO_OK) return rc;
  rc = check_pointers(q, k, v, rel_h, rel_w, out, s);
  if (rc != HALO_OK) return rc;
  const int kind = select_kernel(s);
  if (kind == HALO_KERNEL_NONE) return HALO_ERR_UNSUPPORTED;
  int sm_count = 0;
  rc = device_info(&sm_count);
  if (rc != HALO_OK) return rc;
  if (kind == HALO_KERNEL_TC_BF16) {
    if (const Tc4Entry* e4 = find_tc4(s)) return launch_tc4(*e4, q, k, v, rel_h, rel_w, out, s, sm_count, st);
    if (s.kmask > 0) return HALO_ERR_UNSUPPORTED;  // not reached: select_kernel routes masked shapes to tc4 or simt
    if (const Tc2Entry* e2 = find_tc2(s)) return launch_tc2(*e2, q, k, v, rel_h, rel_w, out, s, sm_count, st);
    if (const Tc3Entry* e3 = find_tc3(s)) return launch_tc3(*e3, q, k, v, rel_h, rel_w, out, s, sm_count, st);
    return launch_tc(*find_tc(s), q, k, v, rel_h, rel_w, out, s, sm_count, st);
  }
  halo::win::Params wp;
  int wthreads = 0, wsmem = 0;
  if (win_plan(s, &wp, &wthreads, &wsmem))
    return (s.dtype == HALO_F32) ? launch_win<float>(q, k, v, rel_h, rel_w, out, s, wp, wthreads, wsmem, st)
                                 : launch_win<__nv_bfloat16>(q, k, v, rel_h, rel_w, out, s, wp, wthreads, wsmem, st);
  cudaError_t err = (s.dtype == HALO_F32) ? launch_simt<float>(q, k, v, rel_h, rel_w, out, s, st)
                                          : launch_simt<__nv_bfloat16>(q, k, v, rel_h, rel_w, out, s, st);
  return err == cudaSuccess ? HALO_OK : HALO_ERR_CUDA;
}

// ----------------------------------------------------------------------------
// Forward with the q, k, v projections inside the kernel (halo_attn_fused)
// ----------------------------------------------------------------------------
using FusedKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap,
                             const halo::fused::Params);
struct FusedEntry {
  int d, win, cin;
  FusedKernel fn;
  int (*smem)(int);
};
template <int D, int WIN, int CIN>
int fused_smem(int xstages) { return halo::fused::smem_bytes<D, WIN, CIN>(xstages); }
#define HALO_FUSED_ENTRY(D, WIN, CIN) \
  FusedEntry { D, WIN, CIN, halo::fused::halo_fused_tc<D, WIN, CIN>, fused_smem<D, WIN, CIN> }
#define HALO_FUSED_WINS(D, CIN)                                                                       \
  HALO_FUSED_ENTRY(D, 8, CIN), HALO_FUSED_ENTRY(D, 10, CIN), HALO_FUSED_ENTRY(D, 12, CIN),            \
      HALO_FUSED_ENTRY(D, 14, CIN)
// (d = 32, c_in = 128 needs more shared memory than a CTA has: the x tiles
// alone are 128 KB next to 144 KB of per-warpgroup tiles and weights)
const FusedEntry kFusedTable[] = {HALO_FUSED_WINS(16, 64), HALO_FUSED_WINS(16, 128), HALO_FUSED_WINS(32, 64)};

const FusedEntry* find_fused(const Shape& s, int c_in) {
  if (s.dtype != HALO_BF16 || s.block != halo::fused::kBlock || s.stride != 1 || (s.H / s.block) % 2)
    return nullptr;
  const int win = s.block + 2 * s.halo;
  for (const FusedEntry& e : kFusedTable)
    if (e.d == s.d && e.win == win && e.cin == c_in) return &e;
  return nullptr;
}

// 4-D map over the NHWC bf16 input map {c_in, W, H, N}; box {64, bw, bh, 1}
// (64 channels = one 128-byte swizzle atom per row).
bool encode_x(CUtensorMap* m, const void* base, const Shape& s, int c_in, int bw, int bh) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  const cuuint64_t C = static_cast<cuuint64_t>(c_in);
  cuuint64_t dims[4] = {C, static_cast<cuuint64_t>(s.W), static_cast<cuuint64_t>(s.H),
                        static_cast<cuuint64_t>(s.N)};
  cuuint64_t strides[3] = {C * 2, C * 2 * s.W, C * 2 * s.W * s.H};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(bw), static_cast<cuuint32_t>(bh), 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over a [rows, c_in] bf16 weight matrix; box {64, d}.
bool encode_w(CUtensorMap* m, const void* base, int rows, int c_in, int d) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(c_in), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(c_in) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(d)};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int attn_fused_device(const void* x, const void* wq, const void* wkv, const void* rel_h, const void* rel_w, void* out,
                      const Shape& s, int c_in, cudaStream_t st) {
  int rc = check_shape(s);
  if (rc != HALO_OK) return rc;
  if (c_in <= 0 || c_in > (1 << 16)) return HALO_ERR_DIMS;
  if (!x || !wq || !wkv || !rel_h || !rel_w || !out) return HALO_ERR_NULL;
  const void* ptrs[6] = {x, wq, wkv, rel_h, rel_w, out};
  for (const void* ptr : ptrs)
    if (reinterpret_cast<uintptr_t>(ptr) % 16) return HALO_ERR_ALIGN;
  if ((static_cast<long long>(c_in) * s.elem()) % 16) return HALO_ERR_ALIGN;
  const size_t xb = static_cast<size_t>(s.N) * s.H * s.W * c_in * s.elem();
  const size_t wb = static_cast<size_t>(s.heads) * s.d * c_in * s.elem();
  const size_t ob = s.out_bytes(), rb = s.rel_bytes();
  if (overlaps(out, ob, x, xb) || overlaps(out, ob, wq, wb) || overlaps(out, ob, wkv, 2 * wb) ||
      overlaps(out, ob, rel_h, rb) || overlaps(out, ob, rel_w, rb))
    return HALO_ERR_ALIAS;
  const FusedEntry* e = find_fused(s, c_in);
  if (!e) return HALO_ERR_UNSUPPORTED;
  int sm_count = 0;
  rc = device_info(&sm_count);
  if (rc != HALO_OK) return rc;
  const int win = s.block + 2 * s.halo;
  CUtensorMap mxq, mxkv, mwq, mwkv;
  if (!encode_x(&mxq, x, s, c_in, halo::fused::kBlock, 2 * halo::fused::kBlock) ||
      !encode_x(&mxkv, x, s, c_in, win, win + halo::fused::kBlock) ||
      !encode_w(&mwq, wq, s.heads * s.d, c_in, s.d) || !encode_w(&mwkv, wkv, 2 * s.heads * s.d, c_in, s.d))
    return HALO_ERR_CUDA;
  cudaFuncAttributes attr;
  if (cudaFuncGetAttributes(&attr, reinterpret_cast<const void*>(e->fn)) != cudaSuccess) return HALO_ERR_CUDA;
  // the setmaxnreg split must fit the launch's registers (see launch_persistent)
  if (256 * halo::fused::kSoftmaxRegs + 128 * halo::fused::kProducerRegs > halo::fused::kThreads * attr.numRegs)
    return HALO_ERR_UNSUPPORTED;
  int optin = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return HALO_ERR_CUDA;
  const int budget = (optin < kMaxDynSmem ? optin : kMaxDynSmem) - static_cast<int>(attr.sharedSizeBytes);
  const int xstages = e->smem(2) <= budget ? 2 : 1;
  const int smem = e->smem(xstages);
  if (smem > budget) return HALO_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(reinterpret_cast<const void*>(e->fn), cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem) != cudaSuccess)
    return HALO_ERR_CUDA;
  halo::fused::Params p;
  p.rel_h = static_cast<const __nv_bfloat16*>(rel_h);
  p.rel_w = static_cast<const __nv_bfloat16*>(rel_w);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.N = s.N;
  p.H = s.H;
  p.W = s.W;
  p.heads = s.heads;
  p.halo = s.halo;
  p.nbx = s.W / halo::fused::kBlock;
  p.npy = s.H / (2 * halo::fused::kBlock);
  const long long pairs = static_cast<long long>(s.N) * p.nbx * p.npy;
  if (pairs * s.heads > 0x7fffffffLL) return HALO_ERR_DIMS;
  p.num_pairs = static_cast<int>(pairs);
  p.xstages = xstages;
  p.c = 1.4426950408889634f / std::sqrt(static_cast<float>(s.d));
  const int grid = static_cast<int>(pairs < sm_count ? pairs : sm_count);
  e->fn<<<grid, halo::fused::kThreads, smem, st>>>(mxq, mxkv, mwq, mwkv, p);
  return cudaGetLastError() == cudaSuccess ? HALO_OK : HALO_ERR_CUDA;
}

// ----------------------------------------------------------------------------
// Backward
// ----------------------------------------------------------------------------
struct BwdPlan {
  halo::bwd::Params p;
  int smem;
  size_t off_dk, off_dv, off_drh, off_drw, ws_bytes;  // workspace layout (bytes)
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

int bwd_plan(const Shape& s, BwdPlan* plan) {
  int rc = check_shape(s);
  if (rc != HALO_OK) return rc;
  if (s.d != 8 && s.d != 16 && s.d != 32 && s.d != 64 && s.d != 128) return HALO_ERR_UNSUPPORTED;
  halo::bwd::Params& p = plan->p;
  p.N = s.N;
  p.H = s.H;
  p.W = s.W;
  p.heads = s.heads;
  p.block = s.block;
  p.halo = s.halo;
  p.stride = s.stride;
  p.kmask = s.kmask;
  p.w = s.block + 2 * s.halo;
  p.R = 2 * p.w - 1;
  p.nqx = s.block / s.stride;
  p.nq = p.nqx * p.nqx;
  p.nbx = s.W / s.block;
  p.nby = s.H / s.block;
  p.c = 1.4426950408889634f / std::sqrt(static_cast<float>(s.d));
  p.s = 1.0f / std::sqrt(static_cast<float>(s.d));
  // largest power-of-two query tile (at most 256) whose item fits in shared memory
  const long long KS = static_cast<long long>(p.w) * p.w;
  if (KS > (1 << 20)) return HALO_ERR_UNSUPPORTED;
  // Row groups per query in the query phase: enough that the tile's queries
  // occupy the CTA's threads (at most one window row per group).
  const int tt = s.d >= 16 ? s.d / 16 : 1;  // threads per (query, row group)
  auto ksplit_for = [&](int qt) {
    const int k = halo::bwd::kThreads / (qt * tt);
    return k < 1 ? 1 : (k > p.w ? p.w : k);
  };
  int qt = 256;
  while (qt > p.nq * 2) qt /= 2;
  for (; qt >= 1; qt /= 2) {
    const int q = qt < p.nq ? qt : p.nq;
    const halo::bwd::Layout L(s.d, static_cast<int>(KS), q, p.w, p.R, ksplit_for(q));
    if (L.bytes() <= kMaxDynSmem) break;
  }
  if (qt < 1) return HALO_ERR_UNSUPPORTED;
  p.QT = qt < p.nq ? qt : p.nq;
  p.ntiles = (p.nq + p.QT - 1) / p.QT;
  p.ksplit = ksplit_for(p.QT);
  plan->smem = halo::bwd::Layout(s.d, static_cast<int>(KS), p.QT, p.w, p.R, p.ksplit).bytes();
  p.num_items = static_cast<long long>(s.N) * p.nby * p.nbx * s.heads * p.ntiles;
  const size_t nin = static_cast<size_t>(s.N) * s.H * s.W * s.heads * s.d;
  const size_t ntab = static_cast<size_t>(p.R) * s.d;
  plan->off_dk = 0;
  plan->off_dv = align256(nin * 4);
  plan->off_drh = plan->off_dv + align256(nin * 4);
  plan->off_drw = plan->off_drh + align256(ntab * 4);
  plan->ws_bytes = plan->off_drw + align256(ntab * 4);
  return HALO_OK;
}

template <typename T, int D>
int launch_bwd_t(const BwdPlan& plan, const void* const* in, void* const* grads, void* ws, int sm_count,
                 cudaStream_t st) {
  auto fn = halo::bwd::halo_bwd_simt<T, D>;
  if (cudaFuncSetAttribute(reinterpret_cast<const void*>(fn), cudaFuncAttributeMaxDynamicSharedMemorySize,
                           plan.smem) != cudaSuccess)
    return HALO_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, halo::bwd::kThreads, plan.smem) != cudaSuccess ||
      per_sm < 1)
    return HALO_ERR_UNSUPPORTED;
  halo::bwd::Ptrs<T> g;
  g.q = static_cast<const T*>(in[0]);
  g.k = static_cast<const T*>(in[1]);
  g.v = static_cast<const T*>(in[2]);
  g.rel_h = static_cast<const T*>(in[3]);
  g.rel_w = static_cast<const T*>(in[4]);
  g.out = static_cast<const T*>(in[5]);
  g.dout = static_cast<const T*>(in[6]);
  g.dq = static_cast<T*>(grads[0]);
  char* w = static_cast<char*>(ws);
  g.dk32 = reinterpret_cast<float*>(w + plan.off_dk);
  g.dv32 = reinterpret_cast<float*>(w + plan.off_dv);
  g.drh32 = reinterpret_cast<float*>(w + plan.off_drh);
  g.drw32 = reinterpret_cast<float*>(w + plan.off_drw);
  const long long cap = static_cast<long long>(per_sm) * sm_count;
  const int grid = static_cast<int>(plan.p.num_items < cap ? plan.p.num_items : cap);
  fn<<<grid, halo::bwd::kThreads, plan.smem, st>>>(g, plan.p);
  if (cudaGetLastError() != cudaSuccess) return HALO_ERR_CUDA;
  const long long nin = static_cast<long long>(plan.p.N) * plan.p.H * plan.p.W * plan.p.heads * D;
  const int ntab = plan.p.R * D;
  const long long nmax = nin > ntab ? nin : ntab;
  long long fb = (nmax + 255) / 256;
  if (fb > 8LL * sm_count) fb = 8LL * sm_count;
  halo::bwd::halo_bwd_finalize<T><<<static_cast<int>(fb), 256, 0, st>>>(
      g.dk32, g.dv32, g.drh32, g.drw32, static_cast<T*>(grads[1]), static_cast<T*>(grads[2]),
      static_cast<T*>(grads[3]), static_cast<T*>(grads[4]), nin, ntab);
  return cudaGetLastError() == cudaSuccess ? HALO_OK : HALO_ERR_CUDA;
}

template <typename T>
int launch_bwd(const BwdPlan& plan, int d, const void* const* in, void* const* grads, void* ws, int sm_count,
               cudaStream_t st) {
  switch (d) {
    case 8: return launch_bwd_t<T, 8>(plan, in, grads, ws, sm_count, st);
    case 16: return launch_bwd_t<T, 16>(plan, in, grads, ws, sm_count, st);
    case 32: return launch_bwd_t<T, 32>(plan, in, grads, ws, sm_count, st);
    case 64: return launch_bwd_t<T, 64>(plan, in, grads, ws, sm_count, st);
    case 128: return launch_bwd_t<T, 128>(plan, in, grads, ws, sm_count, st);
    default: return HALO_ERR_UNSUPPORTED;
  }
}

// Tensor-core backward: bf16, block 8, stride 1 or 2, dim_head 16 or 32,
// window 8..14: (d, window, stride) -> instantiation.
using BwdTcKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap,
                             const halo::bwdtc::Params);
struct BwdTcEntry {
  int d, win, stride;
  BwdTcKernel fn;
  int (*smem)(int);
};
template <int D, int WIN, int STRIDE>
int bwdtc_smem(int stages) { return halo::bwdtc::smem_bytes<D, WIN, STRIDE>(stages); }
#define HALO_BWDTC_ENTRY(D, WIN, S) \
  BwdTcEntry { D, WIN, S, halo::bwdtc::halo_bwd_tc<D, WIN, S>, bwdtc_smem<D, WIN, S> }
#define HALO_BWDTC_WINS(D, S) \
  HALO_BWDTC_ENTRY(D, 8, S), HALO_BWDTC_ENTRY(D, 10, S), HALO_BWDTC_ENTRY(D, 12, S), HALO_BWDTC_ENTRY(D, 14, S)
const BwdTcEntry kBwdTcTable[] = {
    HALO_BWDTC_WINS(16, 1), HALO_BWDTC_WINS(32, 1), HALO_BWDTC_WINS(16, 2), HALO_BWDTC_WINS(32, 2),
};

const BwdTcEntry* find_bwdtc(const Shape& s) {
  if (s.dtype != HALO_BF16 || s.block != halo::bwdtc::kBlock) return nullptr;
  const int win = s.block + 2 * s.halo;
  for (const BwdTcEntry& e : kBwdTcTable)
    if (e.d == s.d && e.win == win && e.stride == s.stride) return &e;
  return nullptr;
}

int launch_bwdtc(const BwdTcEntry& e, const BwdPlan& plan, const void* const* in, void* const* grads, void* ws,
                 const Shape& s, int sm_count, cudaStream_t st) {
  const int win = s.block + 2 * s.halo;
  CUtensorMap mq, mk, mv, mdo;
  // dout is at the output resolution: its map covers (H, W) / stride, and a
  // block's box is (8 / stride)^2 output pixels
  Shape so = s;
  so.H = s.H / s.stride;
  so.W = s.W / s.stride;
  const int ob = halo::bwdtc::kBlock / s.stride;
  if (!encode_nhwc(&mq, in[0], s, halo::bwdtc::kBlock, halo::bwdtc::kBlock, s.stride) ||
      !encode_nhwc(&mk, in[1], s, win, win, 1) || !encode_nhwc(&mv, in[2], s, win, win, 1) ||
      !encode_nhwc(&mdo, in[6], so, ob, ob, 1))
    return HALO_ERR_CUDA;
  cudaFuncAttributes attr;
  if (cudaFuncGetAttributes(&attr, reinterpret_cast<const void*>(e.fn)) != cudaSuccess) return HALO_ERR_CUDA;
  int optin = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return HALO_ERR_CUDA;
  const int budget = (optin < kMaxDynSmem ? optin : kMaxDynSmem) - static_cast<int>(attr.sharedSizeBytes);
  int stages = 4;  // the kernel has four stage barriers
  while (stages > 1 && e.smem(stages) > budget) --stages;
  const int smem = e.smem(stages);
  if (smem > budget) return HALO_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(reinterpret_cast<const void*>(e.fn), cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return HALO_ERR_CUDA;
  halo::bwdtc::Params p;
  p.rel_h = static_cast<const __nv_bfloat16*>(in[3]);
  p.rel_w = static_cast<const __nv_bfloat16*>(in[4]);
  p.out = static_cast<const __nv_bfloat16*>(in[5]);
  p.dout = static_cast<const __nv_bfloat16*>(in[6]);
  p.dq = static_cast<__nv_bfloat16*>(grads[0]);
  char* w = static_cast<char*>(ws);
  p.dk32 = reinterpret_cast<float*>(w + plan.off_dk);
  p.dv32 = reinterpret_cast<float*>(w + plan.off_dv);
  p.drh32 = reinterpret_cast<float*>(w + plan.off_drh);
  p.drw32 = reinterpret_cast<float*>(w + plan.off_drw);
  p.N = s.N;
  p.H = s.H;
  p.W = s.W;
  p.heads = s.heads;
  p.halo = s.halo;
  p.nbx = s.W / halo::bwdtc::kBlock;
  p.nby = s.H / halo::bwdtc::kBlock;
  const long long items = static_cast<long long>(s.N) * p.nbx * p.nby * s.heads;
  if (items > 0x7fffffffLL) return HALO_ERR_DIMS;
  p.num_items = static_cast<int>(items);
  p.stages = stages;
  p.kmask = s.kmask;
  p.c = plan.p.c;
  p.s = plan.p.s;
  const int grid = static_cast<int>(items < sm_count ? items : sm_count);
  e.fn<<<grid, halo::bwdtc::kThreads, smem, st>>>(mq, mk, mv, mdo, p);
  if (cudaGetLastError() != cudaSuccess) return HALO_ERR_CUDA;
  const long long nin = static_cast<long long>(s.N) * s.H * s.W * s.heads * s.d;
  const int ntab = plan.p.R * s.d;
  const long long nmax = nin > ntab ? nin : ntab;
  long long fb = (nmax + 255) / 256;
  if (fb > 8LL * sm_count) fb = 8LL * sm_count;
  halo::bwd::halo_bwd_finalize<__nv_bfloat16><<<static_cast<int>(fb), 256, 0, st>>>(
      p.dk32, p.dv32, p.drh32, p.drw32, static_cast<__nv_bfloat16*>(grads[1]), static_cast<__nv_bfloat16*>(grads[2]),
      static_cast<__nv_bfloat16*>(grads[3]), static_cast<__nv_bfloat16*>(grads[4]), nin, ntab);
  return cudaGetLastError() == cudaSuccess ? HALO_OK : HALO_ERR_CUDA;
}

// Shared by the workspace-taking backward entry point (and any variant that
// brings its own scratch): checks, zeroing, the two launches.
int attn_bwd(const void* const* in, void* const* grads, void* ws, size_t ws_bytes, const Shape& s,
             cudaStream_t st) {
  BwdPlan plan;
  int rc = bwd_plan(s, &plan);
  if (rc != HALO_OK) return rc;
  for (int i = 0; i < 7; ++i)
    if (!in[i]) return HALO_ERR_NULL;
  for (int i = 0; i < 5; ++i)
    if (!grads[i]) return HALO_ERR_NULL;
  for (int i = 0; i < 7; ++i)
    if (reinterpret_cast<uintptr_t>(in[i]) % 16) return HALO_ERR_ALIGN;
  for (int i = 0; i < 5; ++i)
    if (reinterpret_cast<uintptr_t>(grads[i]) % 16) return HALO_ERR_ALIGN;
  if (!ws || reinterpret_cast<uintptr_t>(ws) % 256 || ws_bytes < plan.ws_bytes) return HALO_ERR_WORKSPACE;
  // no gradient (or the workspace) may overlap an input or another gradient
  const size_t ib = s.in_bytes(), ob = s.out_bytes(), rb = s.rel_bytes();
  const size_t in_sz[7] = {ib, ib, ib, rb, rb, ob, ob};
  const size_t g_sz[6] = {ib, ib, ib, rb, rb, plan.ws_bytes};
  const void* gp[6] = {grads[0], grads[1], grads[2], grads[3], grads[4], ws};
  for (int a = 0; a < 6; ++a) {
    for (int i = 0; i < 7; ++i)
      if (overlaps(gp[a], g_sz[a], in[i], in_sz[i])) return HALO_ERR_ALIAS;
    for (int b = a + 1; b < 6; ++b)
      if (overlaps(gp[a], g_sz[a], gp[b], g_sz[b])) return HALO_ERR_ALIAS;
  }
  int sm_count = 0;
  rc = device_info(&sm_count);
  if (rc != HALO_OK) return rc;
  if (cudaMemsetAsync(ws, 0, plan.ws_bytes, st) != cudaSuccess) return HALO_ERR_CUDA;
  // at stride 2 only the strided pixels are queries: dq is zero elsewhere
  if (s.stride == 2 && cudaMemsetAsync(grads[0], 0, ib, st) != cudaSuccess) return HALO_ERR_CUDA;
  if (const BwdTcEntry* e = find_bwdtc(s)) return launch_bwdtc(*e, plan, in, grads, ws, s, sm_count, st);
  return s.dtype == HALO_F32 ? launch_bwd<float>(plan, s.d, in, grads, ws, sm_count, st)
                             : launch_bwd<__nv_bfloat16>(plan, s.d, in, grads, ws, sm_count, st);
}

// ----------------------------------------------------------------------------
// Backward with built-in scratch (halo_attn_bwd_noalloc)
// ----------------------------------------------------------------------------
// The backward's float32 accumulators live in this file-scope array instead
// of a caller-provided workspace.  Every device that loads the library holds
// it until the process exits.  Host code may not pass `g_bwd_scratch` itself
// to a kernel (on the host the name is only a stand-in for the device
// object): its device address is fetched once per device with
// cudaGetSymbolAddress, with that device current, and cached here.
static __device__ __align__(256) unsigned char g_bwd_scratch[HALO_BWD_NOALLOC_MAX_WORKSPACE];
void* g_bwd_scratch_addr[kMaxDevices];

int bwd_scratch(void** addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HALO_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_bwd_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_bwd_scratch) != cudaSuccess || !ptr) return HALO_ERR_CUDA;
    g_bwd_scratch_addr[dev] = ptr;
  }
  *addr = g_bwd_scratch_addr[dev];
  return HALO_OK;
}

// The self test's own result flag: a timeout that a real halo_attn recorded
// in g_halo_error stays there for halo_get_last_error.
__device__ int g_selftest_flag;

__global__ void wait_timeout_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    halo::sm100::mbar_init(&bar, 1);
    halo::sm100::fence_mbar_init();
    // nothing ever arrives on `bar`: the wait must end by its time limit
    g_selftest_flag = halo::sm100::mbar_wait(&bar, 0, limit_ns) ? HALO_OK : HALO_ERR_TIMEOUT;
  }
}

const char* kernel_name_of(const Shape& s) {
  thread_local char name[64];
  const int kind = select_kernel(s);
  if (kind == HALO_KERNEL_NONE) {
    std::snprintf(name, sizeof(name), "none");
  } else if (kind == HALO_KERNEL_TC_BF16) {
    if (const Tc4Entry* e = find_tc4(s))
      std::snprintf(name, sizeof(name), s.kmask > 0 ? "halo_fwd_tc4<%d,%d,masked>" : "halo_fwd_tc4<%d,%d>", e->d,
                    e->win);
    else if (const Tc2Entry* e = find_tc2(s)) std::snprintf(name, sizeof(name), "halo_fwd_tc2<%d,%d>", e->d, e->win);
    else if (const Tc3Entry* e = find_tc3(s))
      std::snprintf(name, sizeof(name), "halo_fwd_tc3<%d,%d,%d>", e->d, e->win, e->block);
    else {
      const TcEntry* t = find_tc(s);
      std::snprintf(name, sizeof(name), "halo_fwd_tc<%d,%d,%d,%d>", t->d, t->win, t->stride, t->parts);
    }
  } else {
    halo::win::Params wp;
    int wthreads = 0, wsmem = 0;
    if (win_plan(s, &wp, &wthreads, &wsmem)) {
      std::snprintf(name, sizeof(name), "halo_fwd_win<%s,%d>", s.dtype == HALO_F32 ? "float" : "bf16", s.d);
    } else {
      const int dmax = s.d <= 16 ? 16 : s.d <= 32 ? 32 : s.d <= 64 ? 64 : 128;
      std::snprintf(name, sizeof(name), "halo_fwd_simt<%s,%d>", s.dtype == HALO_F32 ? "float" : "bf16", dmax);
    }
  }
  return name;
}

}  // namespace

extern "C" {

int halo_attn(const void* q, const void* k, const void* v, const void* rel_h, const void* rel_w, void* out, int N,
              int H, int W, int heads, int dim_head, int block, int halo, int stride, int dtype, void* stream) {
  const Shape s{N, H, W, heads, dim_head, block, halo, stride, dtype};
  return attn_device(q, k, v, rel_h, rel_w, out, s, static_cast<cudaStream_t>(stream));
}

// Two library-owned streams and their events per device, created on first
// use of halo_attn_host: chunk c of the images runs on stream c % 2, so the
// copies of one chunk overlap the kernel and the copies of the previous one.
struct HostPipe {
  bool ready = false;
  cudaStream_t st[2];
  cudaEvent_t ev_in, ev_done[2];
};
HostPipe g_pipe[kMaxDevices];
std::mutex g_pipe_mutex;  // one host thread at a time enqueues through the pipeline streams

int host_pipe(HostPipe** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HALO_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  HostPipe& hp = g_pipe[dev];
  if (!hp.ready) {
    if (cudaStreamCreateWithFlags(&hp.st[0], cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&hp.st[1], cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&hp.ev_in, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&hp.ev_done[0], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&hp.ev_done[1], cudaEventDisableTiming) != cudaSuccess)
      return HALO_ERR_CUDA;
    hp.ready = true;
  }
  *out = &hp;
  return HALO_OK;
}

int halo_attn_host(const void* q_h, const void* k_h, const void* v_h, const void* rel_h_h, const void* rel_w_h,
                   void* out_h, void* q_d, void* k_d, void* v_d, void* rel_h_d, void* rel_w_d, void* out_d, int N,
                   int H, int W, int heads, int dim_head, int block, int halo, int stride, int dtype,
                   void* stream) {
  const Shape s{N, H, W, heads, dim_head, block, halo, stride, dtype};
  int rc = check_shape(s);
  if (rc != HALO_OK) return rc;
  if (!q_h || !k_h || !v_h || !rel_h_h || !rel_w_h || !out_h) return HALO_ERR_NULL;
  rc = check_pointers(q_d, k_d, v_d, rel_h_d, rel_w_d, out_d, s);
  if (rc != HALO_OK) return rc;
  if (select_kernel(s) == HALO_KERNEL_NONE) return HALO_ERR_UNSUPPORTED;
  int sm_count = 0;
  rc = device_info(&sm_count);
  if (rc != HALO_OK) return rc;
  HostPipe* hp = nullptr;
  rc = host_pipe(&hp);
  if (rc != HALO_OK) return rc;
  std::lock_guard<std::mutex> pipe_lock(g_pipe_mutex);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // On an error after the first copy was queued, the caller's stream is still
  // made to wait for everything already queued on the pipeline streams, so
  // that synchronising it before freeing the buffers stays safe.
  auto fail = [&](int code) {
    for (int i = 0; i < 2; ++i)
      if (cudaEventRecord(hp->ev_done[i], hp->st[i]) == cudaSuccess) cudaStreamWaitEvent(st, hp->ev_done[i], 0);
    return code;
  };
  // the tables first, on the caller's stream, then both pipeline streams wait
  // for everything queued on it so far
  const size_t rb = s.rel_bytes();
  if (cudaMemcpyAsync(rel_h_d, rel_h_h, rb, cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(rel_w_d, rel_w_h, rb, cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaEventRecord(hp->ev_in, st) != cudaSuccess || cudaStreamWaitEvent(hp->st[0], hp->ev_in, 0) != cudaSuccess ||
      cudaStreamWaitEvent(hp->st[1], hp->ev_in, 0) != cudaSuccess)
    return fail(HALO_ERR_CUDA);
  // chunks of whole images (NHWC: an image is a contiguous slice of every tensor)
  const int chunks = N < 8 ? N : 8;
  const size_t img_in = s.in_bytes() / N, img_out = s.out_bytes() / N;
  for (int c = 0; c < chunks; ++c) {
    const int n0 = static_cast<int>(static_cast<long long>(N) * c / chunks);
    const int n1 = static_cast<int>(static_cast<long long>(N) * (c + 1) / chunks);
    cudaStream_t cs = hp->st[c & 1];
    const size_t oi = img_in * n0, bi = img_in * (n1 - n0), oo = img_out * n0, bo = img_out * (n1 - n0);
    auto dev = [](void* p, size_t off) { return static_cast<void*>(static_cast<char*>(p) + off); };
    auto host = [](const void* p, size_t off) { return static_cast<const void*>(static_cast<const char*>(p) + off); };
    if (cudaMemcpyAsync(dev(q_d, oi), host(q_h, oi), bi, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
        cudaMemcpyAsync(dev(k_d, oi), host(k_h, oi), bi, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
        cudaMemcpyAsync(dev(v_d, oi), host(v_h, oi), bi, cudaMemcpyHostToDevice, cs) != cudaSuccess)
      return fail(HALO_ERR_CUDA);
    Shape sc = s;
    sc.N = n1 - n0;
    rc = attn_device(dev(q_d, oi), dev(k_d, oi), dev(v_d, oi), rel_h_d, rel_w_d, dev(out_d, oo), sc, cs);
    if (rc != HALO_OK) return fail(rc);
    if (cudaMemcpyAsync(dev(out_h, oo), dev(out_d, oo), bo, cudaMemcpyDeviceToHost, cs) != cudaSuccess)
      return fail(HALO_ERR_CUDA);
  }
  // work queued on the caller's stream after this call waits for both
  if (cudaEventRecord(hp->ev_done[0], hp->st[0]) != cudaSuccess ||
      cudaEventRecord(hp->ev_done[1], hp->st[1]) != cudaSuccess ||
      cudaStreamWaitEvent(st, hp->ev_done[0], 0) != cudaSuccess ||
      cudaStreamWaitEvent(st, hp->ev_done[1], 0) != cudaSuccess)
    return fail(HALO_ERR_CUDA);
  return HALO_OK;
}

int halo_attn_fused(const void* x, const void* wq, const void* wkv, const void* rel_h, const void* rel_w, void* out,
                    int N, int H, int W, int c_in, int heads, int dim_head, int block, int halo, int stride, int dtype,
                    void* stream) {
  const Shape s{N, H, W, heads, dim_head, block, halo, stride, dtype};
  return attn_fused_device(x, wq, wkv, rel_h, rel_w, out, s, c_in, static_cast<cudaStream_t>(stream));
}

const char* halo_fused_kernel_name(int N, int H, int W, int c_in, int heads, int dim_head, int block, int halo,
                                   int stride, int dtype) {
  thread_local char name[64];
  const Shape s{N, H, W, heads, dim_head, block, halo, stride, dtype};
  const FusedEntry* e = (check_shape(s) == HALO_OK) ? find_fused(s, c_in) : nullptr;
  if (e) std::snprintf(name, sizeof(name), "halo_fused_tc<%d,%d,%d>", e->d, e->win, e->cin);
  else std::snprintf(name, sizeof(name), "none");
  return name;
}

int halo_attn_masked(const void* q, const void* k, const void* v, const void* rel_h, const void* rel_w, void* out,
                     int N, int H, int W, int heads, int dim_head, int block, int halo, int stride, int kernel,
                     int dtype, void* stream) {
  Shape s{N, H, W, heads, dim_head, block, halo, stride, dtype};
  s.kmask = kernel;
  if (kernel <= 0) return HALO_ERR_KERNEL;
  return attn_device(q, k, v, rel_h, rel_w, out, s, static_cast<cudaStream_t>(stream));
}

int halo_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* rel_h, const void* rel_w,
                          const void* out, const void* dout, void* dq, void* dk, void* dv, void* drel_h,
                          void* drel_w, int N, int H, int W, int heads, int dim_head, int block, int halo,
                          int stride, int kernel, int dtype, void* stream) {
  Shape s{N, H, W, heads, dim_head, block, halo, stride, dtype};
  s.kmask = kernel;
  BwdPlan plan;
  int rc = bwd_plan(s, &plan);
  if (rc != HALO_OK) return rc;
  if (plan.ws_bytes > HALO_BWD_NOALLOC_MAX_WORKSPACE) return HALO_ERR_SCRATCH_LIMIT;
  void* ws = nullptr;
  rc = bwd_scratch(&ws);
  if (rc != HALO_OK) return rc;
  const void* in[7] = {q, k, v, rel_h, rel_w, out, dout};
  void* grads[5] = {dq, dk, dv, drel_h, drel_w};
  return attn_bwd(in, grads, ws, HALO_BWD_NOALLOC_MAX_WORKSPACE, s, static_cast<cudaStream_t>(stream));
}

int halo_attn_bwd_workspace_size(int N, int H, int W, int heads, int dim_head, int block, int halo, int stride,
                                 int kernel, int dtype, size_t* bytes) {
  if (!bytes) return HALO_ERR_NULL;
  Shape s{N, H, W, heads, dim_head, block, halo, stride, dtype};
  s.kmask = kernel;
  BwdPlan plan;
  const int rc = bwd_plan(s, &plan);
  if (rc != HALO_OK) return rc;
  *bytes = plan.ws_bytes;
  return HALO_OK;
}

int halo_attn_bwd(const void* q, const void* k, const void* v, const void* rel_h, const void* rel_w,
                  const void* out, const void* dout, void* dq, void* dk, void* dv, void* drel_h, void* drel_w,
                  void* workspace, size_t workspace_bytes, int N, int H, int W, int heads, int dim_head, int block,
                  int halo, int stride, int kernel, int dtype, void* stream) {
  Shape s{N, H, W, heads, dim_head, block, halo, stride, dtype};
  s.kmask = kernel;
  const void* in[7] = {q, k, v, rel_h, rel_w, out, dout};
  void* grads[5] = {dq, dk, dv, drel_h, drel_w};
  return attn_bwd(in, grads, workspace, workspace_bytes, s, static_cast<cudaStream_t>(stream));
}

int halo_kernel_for(int N, int H, int W, int heads, int dim_head, int block, int halo, int stride, int dtype) {
  const Shape s{N, H, W, heads, dim_head, block, halo, stride, dtype};
  return select_kernel(s);
}

const char* halo_kernel_name(int N, int H, int W, int heads, int dim_head, int block, int halo, int stride,
                             int dtype) {
  const Shape s{N, H, W, heads, dim_head, block, halo, stride, dtype};
  return kernel_name_of(s);
}

const char* halo_bwd_kernel_name(int N, int H, int W, int heads, int dim_head, int block, int halo, int stride,
                                 int kernel, int dtype) {
  thread_local char name[64];
  Shape s{N, H, W, heads, dim_head, block, halo, stride, dtype};
  s.kmask = kernel;
  BwdPlan plan;
  if (bwd_plan(s, &plan) != HALO_OK) {
    std::snprintf(name, sizeof(name), "none");
  } else if (const BwdTcEntry* e = find_bwdtc(s)) {
    if (e->stride == 1)
      std::snprintf(name, sizeof(name), "halo_bwd_tc<%d,%d>", e->d, e->win);
    else
      std::snprintf(name, sizeof(name), "halo_bwd_tc<%d,%d,%d>", e->d, e->win, e->stride);
  } else {
    std::snprintf(name, sizeof(name), "halo_bwd_simt<%s,%d>", s.dtype == HALO_F32 ? "float" : "bf16", s.d);
  }
  return name;
}

const char* halo_masked_kernel_name(int N, int H, int W, int heads, int dim_head, int block, int halo, int stride,
                                    int kernel, int dtype) {
  Shape s{N, H, W, heads, dim_head, block, halo, stride, dtype};
  s.kmask = kernel;
  if (kernel <= 0) return "none";
  return kernel_name_of(s);
}

const char* halo_strerror(int code) { return status_text(code); }

int halo_get_last_error(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return HALO_ERR_CUDA;
  int flag = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbol(&flag, halo::g_halo_error, sizeof(int)) != cudaSuccess) return HALO_ERR_CUDA;
  if (cudaMemcpyToSymbol(halo::g_halo_error, &zero, sizeof(int)) != cudaSuccess) return HALO_ERR_CUDA;
  return flag;
}

int halo_debug_wait_timeout(int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return HALO_ERR_DIMS;
  int sm_count = 0;
  const int rc = device_info(&sm_count);
  if (rc != HALO_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  wait_timeout_kernel<<<1, 32, 0, st>>>(static_cast<unsigned long long>(limit_us) * 1000ull);
  if (cudaGetLastError() != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess) return HALO_ERR_CUDA;
  int flag = 0;
  if (cudaMemcpyFromSymbol(&flag, g_selftest_flag, sizeof(int)) != cudaSuccess) return HALO_ERR_CUDA;
  return flag;
}

int halo_version(void) { return kVersion; }

}  // extern "C"
