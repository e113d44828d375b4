// halo_simt.cuh -- CUDA-core kernel for blocked local self-attention with
// haloing, float32 arithmetic.  It serves float32 inputs (all shapes) and the
// bf16 shapes the tensor-core kernel does not cover.
//
// Operation: see halo.h (HaloNet sections 2.1-2.2, appendix A; blog page's
// RelPosEmb / HaloAttention index conventions).
//
// One warp per (output pixel, head), lane e holding channels e, e + 32, ...
// of the query and of the accumulator.  The warp walks the w x w window of
// its block in row-major order, four keys at a time: the lanes load those
// keys' k, rel_h, rel_w and v channels together (coalesced across the warp,
// four keys' loads in flight), each key's logit is a warp sum, and an online
// softmax (running max, rescaled sum and accumulator) skips keys outside the
// image (and, with the SASA mask on, keys outside the query's k x k square).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace halo {
namespace simt {

constexpr int kThreads = 128;   // four warps, four (pixel, head) pairs
constexpr int kKeysAtOnce = 4;

// Whether window key (kr, kc) is kept for the query at in-block offset
// (qy, qx) under the SASA mask (section 2.2: halo floor(k/2) and a mask that
// keeps the k x k keys centred on the query): |kr - (qy + halo)| <= kmask/2
// and the same for columns.  kmask 0 keeps every key (HaloNet's own form).
// Image bounds are checked separately.
__device__ __forceinline__ bool sasa_kept(int kr, int kc, int qy, int qx, int halo, int kmask) {
  if (kmask <= 0) return true;
  const int r = kmask >> 1;
  const int dy = kr - qy - halo, dx = kc - qx - halo;
  return dy <= r && dy >= -r && dx <= r && dx >= -r;
}

__device__ __forceinline__ float load_f(const float* p) { return __ldg(p); }
__device__ __forceinline__ float load_f(const __nv_bfloat16* p) { return __bfloat162float(__ldg(p)); }
__device__ __forceinline__ void store_f(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_f(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

template <typename T, int DMAX>
__global__ void __launch_bounds__(kThreads)
    halo_fwd_simt(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const T* __restrict__ rel_h, const T* __restrict__ rel_w, T* __restrict__ out, int N, int H,
                  int W, int heads, int d, int block, int halo, int stride, int kmask, float scale) {
  constexpr int NC = (DMAX + 31) / 32;  // channels per lane
  const int OH = H / stride, OW = W / stride;
  const long long total = static_cast<long long>(N) * OH * OW * heads;
  const long long u = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (u >= total) return;  // uniform across the warp
  long long t = u;
  const int head = static_cast<int>(t % heads);
  t /= heads;
  const int ox = static_cast<int>(t % OW);
  t /= OW;
  const int oy = static_cast<int>(t % OH);
  const int n = static_cast<int>(t / OH);

  const int C = heads * d;
  const int w = block + 2 * halo;
  const int y = stride * oy, x = stride * ox;
  const int by = y / block, bx = x / block;
  const int qy = y - by * block, qx = x - bx * block;
  const int y0 = by * block - halo, x0 = bx * block - halo;

  float qv[NC], acc[NC];
  const T* qp = q + ((static_cast<size_t>(n) * H + y) * W + x) * C + static_cast<size_t>(head) * d;
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const int e = lane + 32 * c;
    qv[c] = (e < d) ? load_f(qp + e) * scale : 0.f;
    acc[c] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int nkeys = w * w;
  for (int kb = 0; kb < nkeys; kb += kKeysAtOnce) {
    float kz[kKeysAtOnce][NC], vv[kKeysAtOnce][NC];
    bool valid[kKeysAtOnce];
#pragma unroll
    for (int g = 0; g < kKeysAtOnce; ++g) {
      const int key = kb + g, kr = key / w, kc = key - (key / w) * w;
      const int Y = y0 + kr, X = x0 + kc;
      valid[g] = key < nkeys && Y >= 0 && Y < H && X >= 0 && X < W && sasa_kept(kr, kc, qy, qx, halo, kmask);
      const size_t off = valid[g] ? ((static_cast<size_t>(n) * H + Y) * W + X) * C + static_cast<size_t>(head) * d : 0;
      const T* rh = rel_h + static_cast<size_t>(valid[g] ? kr - qy + w - 1 : 0) * d;
      const T* rw = rel_w + static_cast<size_t>(valid[g] ? kc - qx + w - 1 : 0) * d;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const int e = lane + 32 * c;
        const bool use = valid[g] && e < d;
        kz[g][c] = use ? load_f(k + off + e) + load_f(rh + e) + load_f(rw + e) : 0.f;
        vv[g][c] = use ? load_f(v + off + e) : 0.f;
      }
    }
#pragma unroll
    for (int g = 0; g < kKeysAtOnce; ++g) {
      float z = 0.f;
#pragma unroll
      for (int c = 0; c < NC; ++c) z = fmaf(qv[c], kz[g][c], z);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
      if (!valid[g]) continue;  // the same for every lane
      if (z > m) {
        const float corr = expf(m - z);  // 0 on the first key (m = -inf)
        l *= corr;
#pragma unroll
        for (int c = 0; c < NC; ++c) acc[c] *= corr;
        m = z;
      }
      const float pz = expf(z - m);
      l += pz;
#pragma unroll
      for (int c = 0; c < NC; ++c) acc[c] = fmaf(pz, vv[g][c], acc[c]);
    }
  }
  const float inv = 1.0f / l;
  T* op = out + ((static_cast<size_t>(n) * OH + oy) * OW + ox) * C + static_cast<size_t>(head) * d;
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const int e = lane + 32 * c;
    if (e < d) store_f(op + e, acc[c] * inv);
  }
}

}  // namespace simt
}  // namespace halo
