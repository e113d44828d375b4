// halo_bwd.cuh -- backward of blocked local self-attention with haloing
// (HaloNet, "Scaling Local Self-Attention for Parameter Efficient Visual
// Backbones", sections 2.1-2.2 and appendix A; the blog page's RelPosEmb /
// HaloAttention index conventions), float32 arithmetic on the CUDA cores.
//
// Gradients of a loss L with respect to q, k, v, rel_h, rel_w given
// dout = dL/dout.  Per query i of a block and key j of its window, with
// z_ij = s q_i . (k_j + rel_h[a_ij] + rel_w[b_ij]) and p_ij = softmax_j(z_ij)
// over the kept keys (inside the image, and inside the k x k square centred
// on the query when the SASA mask of section 2.2 is on):
//   dp_ij = dout_i . v_j,  D_i = dout_i . out_i,  dz_ij = p_ij (dp_ij - D_i)
//   dq_i  = s sum_j dz_ij (k_j + rel_h[a_ij] + rel_w[b_ij])
//   dk_j += s dz_ij q_i,  dv_j += p_ij dout_i   (every window holding key j)
//   drel_h[a] += s sum_{i,j: a_ij = a} dz_ij q_i, likewise drel_w
// (the tables are shared by all heads, section 2.1, footnote 1).
//
// Work item = one block, one head and a tile of up to QT of its queries.  A
// persistent CTA (256 threads) takes items in turn:
//   * load: the item's K and V window (zero outside the image), its queries'
//     q and dout, as float32 in shared memory; the tables once per CTA.
//   * query phase: D/16 threads per (query, row group) (16 channels each,
//     dot products summed with shuffles); a query's window rows are dealt
//     to ksplit groups (rows g, g + ksplit, ...) so that a tile of few
//     queries (16 in a stride-2 block) still occupies the CTA.  The
//     query's relative logits go to shared memory; pass 1 takes each
//     group's row maximum and sum (online, rescaled only when the maximum
//     moves), merged over the groups in shared memory; pass 2 recomputes
//     p, takes dp and dz and accumulates dq, the row sums of dz (per window
//     row, added at once to dq's rel_h term) and the column sums (for the
//     rel_w terms at the end), both kept in shared memory; the groups' dq
//     parts are summed in shared memory.
//   * table phase: drel_h[a] += s sum over the tile's queries of the row sum
//     at table row a times q, drel_w likewise from the column sums; one
//     thread per table element (no atomics), into the CTA's accumulators.
//   * key phase: D/16 threads per window key, dk and dv of the key in
//     registers, looping over the tile's queries with the saved maximum,
//     1/sum and D; the key's sums are added to float32 accumulators in
//     global memory (atomics: up to four windows hold a key).
// A finalize kernel converts the float32 accumulators to the output dtype.
// No device-side waits: nothing here can hang.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "halo_simt.cuh"

namespace halo {
namespace bwd {

constexpr int kThreads = 256;

struct Params {
  int N, H, W, heads, block, halo, stride, kmask;  // kmask: SASA mask size (0 = none)
  int w, R;           // window side, table rows 2w - 1
  int nqx, nq;        // queries per block row, per block
  int QT, ntiles;     // queries per item, items per (block, head)
  int ksplit;         // thread groups sharing one query's window rows in the query phase
  int nbx, nby;
  long long num_items;
  float c;            // log2(e) / sqrt(d): logits in log2 units
  float s;            // 1 / sqrt(d)
};

template <typename T>
struct Ptrs {
  const T *q, *k, *v, *rel_h, *rel_w, *out, *dout;
  T* dq;
  float *dk32, *dv32, *drh32, *drw32;  // float32 accumulators (zeroed by the host)
};

// Shared-memory layout (floats), the same on host and device.
struct Layout {
  int ks, kv, qs, dos, rh, rw, rlh, rlw, cs, rs, st, drh, drw, ms, dqs, total;
  __host__ __device__ Layout(int D, int KS, int QT, int w, int R, int ksplit) {
    int o = 0;
    ks = o; o += KS * D;
    kv = o; o += KS * D;
    qs = o; o += QT * D;
    dos = o; o += QT * D;
    rh = o; o += R * D;
    rw = o; o += R * D;
    rlh = o; o += QT * w;
    rlw = o; o += QT * w;
    cs = o; o += QT * w;
    rs = o; o += QT * w;   // per (query, window row) sum of dz
    st = o; o += QT * 4;   // m (log2 units), 1/l, D, packed (qy, qx)
    drh = o; o += R * D;
    drw = o; o += R * D;
    ms = o; o += ksplit > 1 ? 2 * kThreads : 0;   // per (query, row group): maximum, sum
    dqs = o; o += ksplit > 1 ? QT * D : 0;        // dq summed over the row groups
    total = o;
  }
  __host__ __device__ int bytes() const { return total * 4; }
};

__device__ __forceinline__ float ld(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(__ldg(p)); }

// Sum over the TT consecutive lanes that share one row.
template <int TT>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
  for (int o = TT / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

using simt::sasa_kept;


template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
    halo_bwd_simt(const Ptrs<T> g, const Params p) {
  constexpr int SL = (D >= 16) ? 16 : D;  // channels per thread
  constexpr int TT = D / SL;              // threads per row
  constexpr int RPP = kThreads / TT;      // rows per pass
  static_assert(D % SL == 0 && (TT & (TT - 1)) == 0 && TT <= 32, "dim_head 8, 16, 32, 64 or 128");
  extern __shared__ float sm[];
  const int w = p.w, R = p.R, KS = w * w, QT = p.QT;
  const int KSPLIT = p.ksplit;
  const Layout L(D, KS, QT, w, R, KSPLIT);
  float* Ks = sm + L.ks;
  float* Vs = sm + L.kv;
  float* Qs = sm + L.qs;
  float* DOs = sm + L.dos;
  float* RH = sm + L.rh;
  float* RW = sm + L.rw;
  float* RLH = sm + L.rlh;
  float* RLW = sm + L.rlw;
  float* CS = sm + L.cs;
  float* RS = sm + L.rs;
  float* ST = sm + L.st;
  float* DRH = sm + L.drh;
  float* DRW = sm + L.drw;
  float* MS = sm + L.ms;
  float* DQS = sm + L.dqs;
  const int tid = threadIdx.x;
  const int C = p.heads * D;
  const float c = p.c, sc = p.s;

  for (int i = tid; i < R * D; i += kThreads) {
    RH[i] = ld(g.rel_h + i);
    RW[i] = ld(g.rel_w + i);
    DRH[i] = 0.f;
    DRW[i] = 0.f;
  }

  for (long long item = blockIdx.x; item < p.num_items; item += gridDim.x) {
    long long t = item;
    const int tile = static_cast<int>(t % p.ntiles);
    t /= p.ntiles;
    const int head = static_cast<int>(t % p.heads);
    t /= p.heads;
    const int bx = static_cast<int>(t % p.nbx);
    t /= p.nbx;
    const int by = static_cast<int>(t % p.nby);
    const int n = static_cast<int>(t / p.nby);
    const int q0 = tile * QT;
    const int qn = (p.nq - q0 < QT) ? p.nq - q0 : QT;  // queries in this item
    const int y0 = by * p.block - p.halo, x0 = bx * p.block - p.halo;
    const int OH = p.H / p.stride, OW = p.W / p.stride;

    __syncthreads();  // the previous item's phases are done with shared memory
    // ---- load the window and the queries (float32)
    for (int idx = tid; idx < KS * D; idx += kThreads) {
      const int j = idx / D, e = idx - j * D;
      const int Y = y0 + j / w, X = x0 + j % w;
      float kk = 0.f, vv = 0.f;
      if (Y >= 0 && Y < p.H && X >= 0 && X < p.W) {
        const size_t off = ((static_cast<size_t>(n) * p.H + Y) * p.W + X) * C + static_cast<size_t>(head) * D + e;
        kk = ld(g.k + off);
        vv = ld(g.v + off);
      }
      Ks[idx] = kk;
      Vs[idx] = vv;
    }
    for (int idx = tid; idx < QT * D; idx += kThreads) {
      const int r = idx / D, e = idx - r * D;
      float qq = 0.f, dd = 0.f;
      if (r < qn) {
        const int iq = q0 + r, oy = by * (p.block / p.stride) + iq / p.nqx, ox = bx * (p.block / p.stride) + iq % p.nqx;
        const int y = oy * p.stride, x = ox * p.stride;
        qq = ld(g.q + ((static_cast<size_t>(n) * p.H + y) * p.W + x) * C + static_cast<size_t>(head) * D + e);
        dd = ld(g.dout + ((static_cast<size_t>(n) * OH + oy) * OW + ox) * C + static_cast<size_t>(head) * D + e);
      }
      Qs[idx] = qq;
      DOs[idx] = dd;
    }
    for (int idx = tid; idx < QT * w; idx += kThreads) CS[idx] = 0.f;
    if (KSPLIT > 1)
      for (int idx = tid; idx < QT * D; idx += kThreads) DQS[idx] = 0.f;
    __syncthreads();

    // ---- query phase: TT threads per (query, row group), KSPLIT row groups
    // per query (window rows kg, kg + KSPLIT, ...), so that few queries (a
    // stride-2 block has 16) still occupy the whole CTA
    const int QPP = kThreads / (TT * KSPLIT);  // queries per pass
    for (int base = 0; base < QT; base += QPP) {
      const int grp = tid / TT;                  // (query, row group) of this thread
      const int r = base + grp / KSPLIT, kg = grp % KSPLIT, sl = tid % TT;
      const bool act = r < qn && grp < QPP * KSPLIT;
      const int rr = act ? r : 0;
      const int iq = q0 + rr;
      const int qy = p.stride * (iq / p.nqx), qx = p.stride * (iq % p.nqx);
      const int oy = by * (p.block / p.stride) + iq / p.nqx, ox = bx * (p.block / p.stride) + iq % p.nqx;
      float qv[SL], dov[SL];
#pragma unroll
      for (int e = 0; e < SL; ++e) {
        qv[e] = Qs[rr * D + sl * SL + e];
        dov[e] = DOs[rr * D + sl * SL + e];
      }
      // Every lane of a warp runs the same number of row iterations (the
      // shuffles of group_sum need the whole warp); a group's iteration past
      // the last window row is computed on row 0 and discarded.
      const int NIT = (w + KSPLIT - 1) / KSPLIT;
      // relative logits of this query (log2 units): rel_h of window row kr
      // and rel_w of window column kr, for this group's indices kr
      for (int it = 0; it < NIT; ++it) {
        const bool rv = kg + it * KSPLIT < w;
        const int kr = rv ? kg + it * KSPLIT : 0;
        const float* th = RH + (kr - qy + w - 1) * D + sl * SL;
        const float* tw = RW + (kr - qx + w - 1) * D + sl * SL;
        float ah = 0.f, aw = 0.f;
#pragma unroll
        for (int e = 0; e < SL; ++e) {
          ah = fmaf(qv[e], th[e], ah);
          aw = fmaf(qv[e], tw[e], aw);
        }
        ah = group_sum<TT>(ah);
        aw = group_sum<TT>(aw);
        if (sl == 0 && act && rv) {
          RLH[r * w + kr] = c * ah;
          RLW[r * w + kr] = c * aw;
        }
      }
      // D = dout . out (the forward output)
      float dd = 0.f;
      {
        const T* op = g.out + ((static_cast<size_t>(n) * OH + oy) * OW + ox) * C + static_cast<size_t>(head) * D + sl * SL;
#pragma unroll
        for (int e = 0; e < SL; ++e) dd = fmaf(dov[e], act ? ld(op + e) : 0.f, dd);
        dd = group_sum<TT>(dd);
      }
      __syncthreads();  // every group's relative logits are in shared memory
      // pass 1: maximum and sum over this group's kept keys
      float m = -INFINITY, l = 0.f;
      for (int it = 0; it < NIT; ++it) {
        const bool rv = kg + it * KSPLIT < w;
        const int kr = rv ? kg + it * KSPLIT : 0;
        const int Y = y0 + kr;
        const bool rin = act && rv && Y >= 0 && Y < p.H;
        const float rlh = RLH[rr * w + kr];
        for (int kc = 0; kc < w; ++kc) {
          const int X = x0 + kc, j = kr * w + kc;
          const float* kp = Ks + j * D + sl * SL;
          float z = 0.f;
#pragma unroll
          for (int e = 0; e < SL; ++e) z = fmaf(qv[e], kp[e], z);
          z = group_sum<TT>(z);
          const bool kept = rin && X >= 0 && X < p.W && sasa_kept(kr, kc, qy, qx, p.halo, p.kmask);
          if (kept) {
            z = fmaf(z, c, rlh + RLW[rr * w + kc]);
            if (z > m) {
              l *= exp2f(m - z);  // 0 on the first kept key
              m = z;
            }
            l += exp2f(z - m);
          }
        }
      }
      if (KSPLIT > 1) {
        // merge the groups' (maximum, sum) pairs of each query
        if (sl == 0) {
          MS[2 * grp] = m;
          MS[2 * grp + 1] = l;
        }
        __syncthreads();
        const int g0 = (grp / KSPLIT) * KSPLIT;
        float mm = -INFINITY;
        for (int u = 0; u < KSPLIT; ++u) mm = fmaxf(mm, MS[2 * (g0 + u)]);
        float ll = 0.f;
        for (int u = 0; u < KSPLIT; ++u) {
          const float mu = MS[2 * (g0 + u)];
          if (mu != -INFINITY) ll += MS[2 * (g0 + u) + 1] * exp2f(mu - mm);
        }
        m = mm;
        l = ll;
      }
      const float inv_l = act ? 1.0f / l : 0.f;
      // pass 2: p, dz; dq and the row / column sums of dz
      float dq[SL];
#pragma unroll
      for (int e = 0; e < SL; ++e) dq[e] = 0.f;
      for (int it = 0; it < NIT; ++it) {
        const bool rv = kg + it * KSPLIT < w;
        const int kr = rv ? kg + it * KSPLIT : 0;
        const int Y = y0 + kr;
        const bool rin = act && rv && Y >= 0 && Y < p.H;
        const float rlh = RLH[rr * w + kr];
        float rowsum = 0.f;
        for (int kc = 0; kc < w; ++kc) {
          const int X = x0 + kc, j = kr * w + kc;
          const float* kp = Ks + j * D + sl * SL;
          const float* vp = Vs + j * D + sl * SL;
          float z = 0.f, dp = 0.f;
#pragma unroll
          for (int e = 0; e < SL; ++e) {
            z = fmaf(qv[e], kp[e], z);
            dp = fmaf(dov[e], vp[e], dp);
          }
          z = group_sum<TT>(z);
          dp = group_sum<TT>(dp);
          const bool kept = rin && X >= 0 && X < p.W && sasa_kept(kr, kc, qy, qx, p.halo, p.kmask);
          const float pr = kept ? exp2f(fmaf(z, c, rlh + RLW[rr * w + kc]) - m) * inv_l : 0.f;
          const float dz = pr * (dp - dd);
#pragma unroll
          for (int e = 0; e < SL; ++e) dq[e] = fmaf(dz, kp[e], dq[e]);
          rowsum += dz;
          if (sl == 0 && act && rv) {
            if (KSPLIT > 1) atomicAdd(&CS[r * w + kc], dz);
            else CS[r * w + kc] += dz;
          }
        }
        if (rin) {
          const int a = kr - qy + w - 1;
          const float* th = RH + a * D + sl * SL;
#pragma unroll
          for (int e = 0; e < SL; ++e) dq[e] = fmaf(rowsum, th[e], dq[e]);
        }
        // the row's dz sum for the drel_h phase (zero for rows outside the image)
        if (sl == 0 && act && rv) RS[r * w + kr] = rin ? rowsum : 0.f;
      }
      if (KSPLIT > 1) {
        if (act) {
#pragma unroll
          for (int e = 0; e < SL; ++e) atomicAdd(&DQS[r * D + sl * SL + e], dq[e]);
        }
        __syncthreads();  // column sums and dq partials complete
      } else {
        __syncwarp();
      }
      // rel_w terms of dq and drel_w: window columns kg, kg + KSPLIT, ...
      if (act) {
        float dw[SL];
#pragma unroll
        for (int e = 0; e < SL; ++e) dw[e] = 0.f;
        for (int kc = kg; kc < w; kc += KSPLIT) {
          const float cs = CS[r * w + kc];
          const int b = kc - qx + w - 1;
          const float* tw = RW + b * D + sl * SL;
#pragma unroll
          for (int e = 0; e < SL; ++e) dw[e] = fmaf(cs, tw[e], dw[e]);
        }
        if (KSPLIT > 1) {
#pragma unroll
          for (int e = 0; e < SL; ++e) atomicAdd(&DQS[r * D + sl * SL + e], dw[e]);
        } else {
#pragma unroll
          for (int e = 0; e < SL; ++e) dq[e] += dw[e];
        }
      }
      if (KSPLIT > 1) {
        __syncthreads();  // every group's rel_w terms are in
        if (act && kg == 0) {
#pragma unroll
          for (int e = 0; e < SL; ++e) dq[e] = DQS[r * D + sl * SL + e];
        }
      }
      if (act && kg == 0) {
        const int y = oy * p.stride, x = ox * p.stride;
        T* dst = g.dq + ((static_cast<size_t>(n) * p.H + y) * p.W + x) * C + static_cast<size_t>(head) * D + sl * SL;
#pragma unroll
        for (int e = 0; e < SL; ++e) simt::store_f(dst + e, sc * dq[e]);
        if (sl == 0) {
          ST[4 * r + 0] = m;
          ST[4 * r + 1] = inv_l;
          ST[4 * r + 2] = dd;
          ST[4 * r + 3] = __int_as_float((qy << 16) | qx);
        }
      }
      __syncthreads();  // the next pass reuses the merge buffer
    }
    __syncthreads();

    // ---- table phase: drel_h[a] += s sum over the tile's queries of the dz
    // sum of the window row at index a, times q; drel_w likewise with the
    // column sums.  One thread per table element: no atomics.
    for (int idx = tid; idx < 2 * R * D; idx += kThreads) {
      const bool wcol = idx >= R * D;
      const int ae = wcol ? idx - R * D : idx, a = ae / D, e = ae - a * D;
      const float* sums = wcol ? CS : RS;
      float acc = 0.f;
      for (int i = 0; i < qn; ++i) {
        const int qyx = __float_as_int(ST[4 * i + 3]);
        // table row a = kr - qy + w - 1 (rel_h), a = kc - qx + w - 1 (rel_w)
        const int kr = a + (wcol ? (qyx & 0xffff) : (qyx >> 16)) - (w - 1);
        if (kr >= 0 && kr < w) acc = fmaf(sums[i * w + kr], Qs[i * D + e], acc);
      }
      (wcol ? DRW : DRH)[ae] += sc * acc;
    }

    // ---- key phase
    for (int base = 0; base < KS; base += RPP) {
      const int j = base + tid / TT, sl = tid % TT;
      const bool inkey = j < KS;
      const int jj = inkey ? j : 0;
      const int kr = jj / w, kc = jj % w;
      const int Y = y0 + kr, X = x0 + kc;
      const bool kin = inkey && Y >= 0 && Y < p.H && X >= 0 && X < p.W;
      float kv[SL], vv[SL], dk[SL], dv[SL];
#pragma unroll
      for (int e = 0; e < SL; ++e) {
        kv[e] = Ks[jj * D + sl * SL + e];
        vv[e] = Vs[jj * D + sl * SL + e];
        dk[e] = 0.f;
        dv[e] = 0.f;
      }
      for (int i = 0; i < qn; ++i) {
        const float* qp = Qs + i * D + sl * SL;
        const float* dp_ = DOs + i * D + sl * SL;
        float z = 0.f, dp = 0.f;
#pragma unroll
        for (int e = 0; e < SL; ++e) {
          z = fmaf(kv[e], qp[e], z);
          dp = fmaf(vv[e], dp_[e], dp);
        }
        z = group_sum<TT>(z);
        dp = group_sum<TT>(dp);
        const int qyx = __float_as_int(ST[4 * i + 3]);
        const bool kept = kin && sasa_kept(kr, kc, qyx >> 16, qyx & 0xffff, p.halo, p.kmask);
        const float pr = kept ? exp2f(fmaf(z, c, RLH[i * w + kr] + RLW[i * w + kc]) - ST[4 * i]) * ST[4 * i + 1] : 0.f;
        const float dz = pr * (dp - ST[4 * i + 2]);
#pragma unroll
        for (int e = 0; e < SL; ++e) {
          dv[e] = fmaf(pr, dp_[e], dv[e]);
          dk[e] = fmaf(dz, qp[e], dk[e]);
        }
      }
      if (kin) {
        const size_t off = ((static_cast<size_t>(n) * p.H + Y) * p.W + X) * C + static_cast<size_t>(head) * D + sl * SL;
#pragma unroll
        for (int e = 0; e < SL; e += 4) {
          atomicAdd(reinterpret_cast<float4*>(g.dk32 + off + e),
                    make_float4(sc * dk[e], sc * dk[e + 1], sc * dk[e + 2], sc * dk[e + 3]));
          atomicAdd(reinterpret_cast<float4*>(g.dv32 + off + e), make_float4(dv[e], dv[e + 1], dv[e + 2], dv[e + 3]));
        }
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < R * D; i += kThreads) {
    atomicAdd(g.drh32 + i, DRH[i]);
    atomicAdd(g.drw32 + i, DRW[i]);
  }
}

// float32 accumulators -> the output dtype.
template <typename T>
__global__ void halo_bwd_finalize(const float* __restrict__ dk32, const float* __restrict__ dv32,
                                  const float* __restrict__ drh32, const float* __restrict__ drw32, T* dk, T* dv,
                                  T* drh, T* drw, long long n_in, int n_tab) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long n = n_in > n_tab ? n_in : n_tab;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    if (i < n_in) {
      simt::store_f(dk + i, dk32[i]);
      simt::store_f(dv + i, dv32[i]);
    }
    if (i < n_tab) {
      simt::store_f(drh + i, drh32[i]);
      simt::store_f(drw + i, drw32[i]);
    }
  }
}

}  // namespace bwd
}  // namespace halo
