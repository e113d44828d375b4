// halo_win.cuh -- CUDA-core kernel for blocked local self-attention with
// haloing, float32 arithmetic, one block's window staged once in shared
// memory (HaloNet, "Scaling Local Self-Attention for Parameter Efficient
// Visual Backbones", sections 2.1-2.2 and appendix A; the blog page's
// RelPosEmb / HaloAttention index conventions).
//
// The method's point (section 2.2): neighbouring queries share most of their
// neighbourhood, so a block's window is extracted once for all its queries.
// Work item = one block and one head (CTA): the w x w window of k and v
// (zero outside the image) and both relative tables go to shared memory as
// float32; then TT threads per query (SL channels each; dot products summed
// with shuffles) walk the window with an online softmax.  Every thread of a
// warp reads the same key at the same time (shared-memory broadcast), so each
// key costs 2 SL fused multiply-adds per thread and one exponential per query.
// Each query's relative logits q.rel_h[kr - qy + w - 1] and
// q.rel_w[kc - qx + w - 1] are taken once (2w dot products) and kept in
// shared memory.  The softmax offset is a per-query upper bound of the largest
// logit (|q| max|k| plus the largest relative logits), so a row takes one pass
// without rescaling; the online softmax remains for rows where the bound could
// lie too far above the maximum.  Optional SASA mask (section 2.2): keys
// outside the query's k x k square are skipped.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "halo_simt.cuh"

namespace halo {
namespace win {

constexpr int kMaxThreads = 256;

struct Params {
  int N, H, W, heads, block, halo, stride, kmask;
  int w, nqx, nq, nbx, nby;
  int qpass;     // queries per pass of the CTA
  float c;       // log2(e) / sqrt(d): logits in log2 units
};

// Shared-memory floats for one item (the last 8: per-warp maxima of |k|).
__host__ __device__ inline int smem_floats(int D, int w, int qpass) {
  const int KS = w * w, R = 2 * w - 1;
  return 2 * KS * D + 2 * R * D + 2 * qpass * w + 8;
}

__device__ __forceinline__ float ldf(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ldf(const __nv_bfloat16* p) { return __bfloat162float(__ldg(p)); }

template <int TT>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
  for (int o = TT / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <typename T, int D>
__global__ void __launch_bounds__(kMaxThreads)
    halo_fwd_win(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                 const T* __restrict__ rel_h, const T* __restrict__ rel_w, T* __restrict__ out, const Params p) {
  constexpr int SL = (D >= 16) ? 16 : D;  // channels per thread
  constexpr int TT = D / SL;              // threads per query
  static_assert(D % SL == 0 && (TT & (TT - 1)) == 0 && TT <= 32, "dim_head 8, 16, 32, 64 or 128");
  extern __shared__ float sm[];
  const int w = p.w, KS = w * w, R = 2 * w - 1;
  float* Ks = sm;
  float* Vs = Ks + KS * D;
  float* RH = Vs + KS * D;
  float* RW = RH + R * D;
  float* RL = RW + R * D;  // per query of the pass: w rel_h logits, then w rel_w logits
  float* KM = RL + 2 * p.qpass * w;  // per-warp maxima of |k| over the window
  const int C = p.heads * D;
  const int tid = threadIdx.x, nthr = blockDim.x;

  long long t = blockIdx.x;
  const int head = static_cast<int>(t % p.heads);
  t /= p.heads;
  const int bx = static_cast<int>(t % p.nbx);
  t /= p.nbx;
  const int by = static_cast<int>(t % p.nby);
  const int n = static_cast<int>(t / p.nby);
  const int y0 = by * p.block - p.halo, x0 = bx * p.block - p.halo;
  const int OH = p.H / p.stride, OW = p.W / p.stride;

  // ---- the window of k and v, and the tables (float32)
  for (int idx = tid; idx < KS * (D / 4); idx += nthr) {
    const int j = idx / (D / 4), e = (idx - j * (D / 4)) * 4;
    const int Y = y0 + j / w, X = x0 + j % w;
    float4 kk = make_float4(0.f, 0.f, 0.f, 0.f), vv = kk;
    if (Y >= 0 && Y < p.H && X >= 0 && X < p.W) {
      const size_t off = ((static_cast<size_t>(n) * p.H + Y) * p.W + X) * C + static_cast<size_t>(head) * D + e;
      kk = make_float4(ldf(k + off), ldf(k + off + 1), ldf(k + off + 2), ldf(k + off + 3));
      vv = make_float4(ldf(v + off), ldf(v + off + 1), ldf(v + off + 2), ldf(v + off + 3));
    }
    *reinterpret_cast<float4*>(Ks + j * D + e) = kk;
    *reinterpret_cast<float4*>(Vs + j * D + e) = vv;
  }
  for (int idx = tid; idx < R * D; idx += nthr) {
    RH[idx] = ldf(rel_h + idx);
    RW[idx] = ldf(rel_w + idx);
  }
  __syncthreads();
  // the largest key norm of the window (zero keys outside the image)
  {
    float km = 0.f;
    for (int j = tid; j < KS; j += nthr) {
      float s2 = 0.f;
#pragma unroll
      for (int e = 0; e < D; ++e) s2 = fmaf(Ks[j * D + e], Ks[j * D + e], s2);
      km = fmaxf(km, s2);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) km = fmaxf(km, __shfl_xor_sync(0xffffffffu, km, o));
    if ((tid & 31) == 0) KM[tid >> 5] = km;
    __syncthreads();
  }
  float kmax = 0.f;
  for (int i = 0; i < (nthr + 31) / 32; ++i) kmax = fmaxf(kmax, KM[i]);
  kmax = sqrtf(kmax);

  const float c = p.c;
  const int r_kept = p.kmask > 0 ? (p.kmask >> 1) : (1 << 20);
  for (int base = 0; base < p.nq; base += p.qpass) {
    const int rl = tid / TT, sl = tid % TT;  // query of this pass, channel slice
    const int iq = base + rl;
    const bool act = rl < p.qpass && iq < p.nq;
    const int iqs = act ? iq : 0;
    const int oy = by * p.nqx + iqs / p.nqx, ox = bx * p.nqx + iqs % p.nqx;
    const int y = oy * p.stride, x = ox * p.stride;
    const int qy = y - by * p.block, qx = x - bx * p.block;
    float qv[SL], acc[SL];
    {
      const T* qp = q + ((static_cast<size_t>(n) * p.H + y) * p.W + x) * C + static_cast<size_t>(head) * D + sl * SL;
#pragma unroll
      for (int e = 0; e < SL; ++e) {
        qv[e] = act ? ldf(qp + e) * c : 0.f;
        acc[e] = 0.f;
      }
    }
    float* rlq = RL + (act ? rl : 0) * 2 * w;
    for (int i = 0; i < w; ++i) {
      const float* th = RH + (i - qy + w - 1) * D + sl * SL;
      const float* tw = RW + (i - qx + w - 1) * D + sl * SL;
      float ah = 0.f, aw = 0.f;
#pragma unroll
      for (int e = 0; e < SL; ++e) {
        ah = fmaf(qv[e], th[e], ah);
        aw = fmaf(qv[e], tw[e], aw);
      }
      ah = group_sum<TT>(ah);
      aw = group_sum<TT>(aw);
      if (sl == 0 && act) {
        rlq[i] = ah;
        rlq[w + i] = aw;
      }
    }
    __syncwarp();
    // The softmax offset.  An upper bound of the row's largest logit:
    // |q c| max|k| (Cauchy-Schwarz) plus the largest relative logits; the
    // query's own pixel (always a kept key) gives a lower bound.  While the
    // two are within 100 (log2 units) every p = 2^(z - m) stays a normal
    // float and the largest is at least 2^-100, so one pass with this fixed m
    // loses nothing; otherwise the online softmax (running maximum, rescaled
    // sums) takes the row.
    float qn2 = 0.f;
#pragma unroll
    for (int e = 0; e < SL; ++e) qn2 = fmaf(qv[e], qv[e], qn2);
    qn2 = group_sum<TT>(qn2);
    float mh = -INFINITY, mw = -INFINITY;
    for (int i = 0; i < w; ++i) {
      mh = fmaxf(mh, rlq[i]);
      mw = fmaxf(mw, rlq[w + i]);
    }
    const float m_ub = sqrtf(qn2) * kmax + mh + mw;
    float z_self;
    {
      const int js = (qy + p.halo) * w + qx + p.halo;
      const float* kp = Ks + js * D + sl * SL;
      float z = 0.f;
#pragma unroll
      for (int e = 0; e < SL; ++e) z = fmaf(qv[e], kp[e], z);
      z_self = group_sum<TT>(z) + rlq[qy + p.halo] + rlq[w + qx + p.halo];
    }
    const bool bounded = m_ub - z_self <= 100.0f;
    float m = bounded ? m_ub : -INFINITY, l = 0.f;
    for (int kr = 0; kr < w; ++kr) {
      const int Y = y0 + kr;
      const bool rin = Y >= 0 && Y < p.H && kr - qy - p.halo <= r_kept && qy + p.halo - kr <= r_kept;
      const float zr = rlq[kr];
      for (int kc = 0; kc < w; ++kc) {
        const int X = x0 + kc, j = kr * w + kc;
        const float* kp = Ks + j * D + sl * SL;
        float z0 = 0.f, z1 = 0.f;
#pragma unroll
        for (int e = 0; e < SL; e += 2) {
          z0 = fmaf(qv[e], kp[e], z0);
          z1 = fmaf(qv[e + 1], kp[e + 1], z1);
        }
        const float z = group_sum<TT>(z0 + z1) + zr + rlq[w + kc];
        const bool kept = rin && X >= 0 && X < p.W && kc - qx - p.halo <= r_kept && qx + p.halo - kc <= r_kept;
        if (kept) {  // the same for every thread of a query's group
          if (!bounded && z > m) {
            const float corr = exp2f(m - z);  // 0 on the first kept key
            l *= corr;
#pragma unroll
            for (int e = 0; e < SL; ++e) acc[e] *= corr;
            m = z;
          }
          const float pz = exp2f(z - m);
          l += pz;
          const float* vp = Vs + j * D + sl * SL;
#pragma unroll
          for (int e = 0; e < SL; ++e) acc[e] = fmaf(pz, vp[e], acc[e]);
        }
      }
    }
    if (act) {
      const float inv = 1.0f / l;
      T* op = out + ((static_cast<size_t>(n) * OH + oy) * OW + ox) * C + static_cast<size_t>(head) * D + sl * SL;
#pragma unroll
      for (int e = 0; e < SL; ++e) simt::store_f(op + e, acc[e] * inv);
    }
    __syncwarp();
  }
}

}  // namespace win
}  // namespace halo
