// halo_simt.cuh -- CUDA-core kernel for blocked local self-attention with
// haloing, float32 arithmetic.  It serves float32 inputs (all shapes) and the
// bf16 shapes the tensor-core kernel does not cover.
//
// Operation: see halo.h (HaloNet sections 2.1-2.2, appendix A; blog page's
// RelPosEmb / HaloAttention index conventions).
//
// One thread per (output pixel, head).  The thread keeps its query in
// registers, walks the w x w window of its block in row-major order with an
// online softmax (running max, rescaled sum and accumulator), skipping keys
// outside the image, and writes d outputs.  Threads of a warp cover
// consecutive (pixel, head) pairs, so their K/V reads are contiguous channels.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace halo {
namespace simt {

constexpr int kThreads = 128;

__device__ __forceinline__ float load_f(const float* p) { return __ldg(p); }
__device__ __forceinline__ float load_f(const __nv_bfloat16* p) { return __bfloat162float(__ldg(p)); }
__device__ __forceinline__ void store_f(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_f(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

template <typename T, int DMAX>
__global__ void __launch_bounds__(kThreads)
    halo_fwd_simt(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const T* __restrict__ rel_h, const T* __restrict__ rel_w, T* __restrict__ out, int N, int H,
                  int W, int heads, int d, int block, int halo, int stride, float scale) {
  const int OH = H / stride, OW = W / stride;
  const long long total = static_cast<long long>(N) * OH * OW * heads;
  const long long u = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (u >= total) return;
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

  float qv[DMAX];
  float acc[DMAX];
  const T* qp = q + ((static_cast<size_t>(n) * H + y) * W + x) * C + static_cast<size_t>(head) * d;
#pragma unroll
  for (int e = 0; e < DMAX; ++e) {
    qv[e] = (e < d) ? load_f(qp + e) * scale : 0.f;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int kr = 0; kr < w; ++kr) {
    const int Y = y0 + kr;
    if (Y < 0 || Y >= H) continue;
    const T* rh = rel_h + static_cast<size_t>(kr - qy + w - 1) * d;
    for (int kc = 0; kc < w; ++kc) {
      const int X = x0 + kc;
      if (X < 0 || X >= W) continue;
      const T* rw = rel_w + static_cast<size_t>(kc - qx + w - 1) * d;
      const size_t off = ((static_cast<size_t>(n) * H + Y) * W + X) * C + static_cast<size_t>(head) * d;
      float z = 0.f;
#pragma unroll
      for (int e = 0; e < DMAX; ++e)
        if (e < d) z = fmaf(qv[e], load_f(k + off + e) + load_f(rh + e) + load_f(rw + e), z);
      if (z > m) {
        const float corr = expf(m - z);  // 0 on the first key (m = -inf)
        l *= corr;
#pragma unroll
        for (int e = 0; e < DMAX; ++e) acc[e] *= corr;
        m = z;
      }
      const float pz = expf(z - m);
      l += pz;
#pragma unroll
      for (int e = 0; e < DMAX; ++e)
        if (e < d) acc[e] = fmaf(pz, load_f(v + off + e), acc[e]);
    }
  }
  const float inv = 1.0f / l;
  T* op = out + ((static_cast<size_t>(n) * OH + oy) * OW + ox) * C + static_cast<size_t>(head) * d;
#pragma unroll
  for (int e = 0; e < DMAX; ++e)
    if (e < d) store_f(op + e, acc[e] * inv);
}

}  // namespace simt
}  // namespace halo
