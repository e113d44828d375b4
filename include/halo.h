/*
 * halo.h -- C ABI of libhalo: HaloNet blocked local self-attention with
 * haloing on NVIDIA B200 (sm_100a).
 *
 * The operation ("Scaling Local Self-Attention for Parameter Efficient Visual
 * Backbones", sections 2.1-2.2, Figures 1-2, Appendix A; the blog page's
 * HaloAttention / RelPosEmb modules for the concrete index conventions):
 *
 *   The H x W map is cut into non-overlapping block x block query blocks.
 *   Block (by, bx) attends to the w x w window (w = block + 2*halo) whose top
 *   left pixel is (by*block - halo, bx*block - halo); window keys outside the
 *   image are removed from the softmax.  For query pixel (y, x) with in-block
 *   offset (qy, qx) and window key (kr, kc) at image pixel (Y, X), per head:
 *
 *     z = s * q[y,x] . ( k[Y,X] + rel_h[kr - qy + w - 1] + rel_w[kc - qx + w - 1] )
 *     out[y/stride, x/stride] = sum_keys softmax(z) * v[Y,X]          s = dim_head^-1/2
 *
 *   stride 2 takes the queries at even in-block offsets (0, 2, .., block-2)
 *   and keeps the stride-1 window (section 2.2, Figure 2).
 *
 * Layouts (all row-major, contiguous, no padding):
 *   q, k, v : [N, H, W, heads*dim_head]  (NHWC; channel = head*dim_head + e)
 *   rel_h, rel_w : [2*w - 1, dim_head]   (shared by all heads)
 *   out     : [N, H/stride, W/stride, heads*dim_head]
 *
 * Conventions shared by every entry point:
 *   - Return value: HALO_OK (0) or a negative halo_status code; nothing is
 *     launched when an argument check fails.
 *   - Device-pointer calls are asynchronous on `stream` (a cudaStream_t; NULL
 *     means the legacy default stream).  The library allocates no device
 *     memory for them and keeps no pointer after the call returns.  The caller
 *     owns every buffer and must keep it alive until the stream work is done.
 *   - `out` must not overlap any input.
 *   - Thread safety: calls from several host threads are safe.  TMA
 *     descriptors are encoded on the host for every call (kernel parameters);
 *     the only process-wide state is a mutex-guarded table of per-device
 *     properties and the driver entry point used for the encoding.
 */
#ifndef HALO_H_
#define HALO_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HALO_F32 = 0,  /* float32 inputs and output, float32 arithmetic */
  HALO_BF16 = 1  /* bfloat16 inputs and output, float32 accumulation */
} halo_dtype_t;

typedef enum {
  HALO_OK = 0,
  HALO_ERR_NULL = -1,          /* a required pointer is NULL */
  HALO_ERR_DIMS = -2,          /* a size is non-positive, or too large */
  HALO_ERR_DIVISIBILITY = -3,  /* H or W not a multiple of block, or block not a multiple of stride */
  HALO_ERR_STRIDE = -4,        /* stride not 1 or 2 */
  HALO_ERR_ALIGN = -5,         /* a pointer is not 16-byte aligned, or a row of C channels is not a multiple of 16 bytes */
  HALO_ERR_UNSUPPORTED = -6,   /* a shape no kernel of this library handles (see halo_kernel_for) */
  HALO_ERR_CUDA = -7,          /* a CUDA runtime call or kernel launch failed */
  HALO_ERR_TIMEOUT = -8,       /* a bounded device-side wait ran out (reported by halo_get_last_error) */
  HALO_ERR_DTYPE = -9,         /* dtype is not a halo_dtype_t value */
  HALO_ERR_ALIAS = -10,        /* out overlaps an input */
  HALO_ERR_DEVICE = -11,       /* the current device is not an sm_100 GPU */
  HALO_ERR_KERNEL = -12,       /* SASA mask size not odd, or larger than 2*halo+1 */
  HALO_ERR_WORKSPACE = -13,    /* the backward's workspace is NULL, not 256-byte aligned or too small */
  HALO_ERR_SCRATCH_LIMIT = -14 /* halo_attn_bwd_noalloc: the shape needs more than its built-in scratch */
} halo_status;

/* Which kernel halo_attn would launch for a shape (halo_kernel_for). */
typedef enum {
  HALO_KERNEL_NONE = 0,       /* the shape is rejected */
  HALO_KERNEL_SIMT_F32 = 1,   /* CUDA-core kernel (float32 arithmetic); all float32 shapes, and bf16 shapes the tensor-core kernel does not cover */
  HALO_KERNEL_TC_BF16 = 2     /* TMA + tcgen05/TMEM tensor-core kernel for bf16 */
} halo_kernel_t;

/*
 * halo_attn -- the fused operation on device buffers.
 *
 * q, k, v, rel_h, rel_w, out: device pointers in the layouts above, all of
 * dtype `dtype`, each 16-byte aligned.  N, H, W, heads, dim_head, block > 0,
 * halo >= 0 (halo 0 is attention on isolated blocks, section 4.3),
 * H % block == 0, W % block == 0, stride in {1, 2}, block % stride == 0.
 * heads*dim_head*sizeof(dtype) must be a multiple of 16 bytes.
 *
 * Asynchronous: returns after the launch is queued on `stream`.  Errors found
 * by the device (a bounded wait that ran out) are recorded in a device flag
 * that halo_get_last_error() reads.
 */
int halo_attn(const void* q, const void* k, const void* v, const void* rel_h, const void* rel_w, void* out,
              int N, int H, int W, int heads, int dim_head, int block, int halo, int stride, int dtype,
              void* stream);

/*
 * halo_attn_host -- the same operation on HOST buffers (end-to-end form).
 *
 * q_h .. rel_w_h: host input pointers (pinned memory is needed for the copies
 * to overlap), out_h: host output pointer.  q_d .. out_d: caller-owned device
 * buffers of the same sizes that the call uses as staging; the library
 * allocates no memory.  The call splits the batch into up to 8 chunks of
 * whole images and queues, per chunk, the host->device copies of its q, k, v,
 * the kernel on it and the device->host copy of its output, alternating
 * between two library-owned streams (created once per device on first use),
 * so that one chunk's copies overlap the previous chunk's kernel and copies.
 * The work is ordered after everything queued on `stream` before the call,
 * and work queued on `stream` after the call waits for all of it; the call
 * returns without waiting: synchronise `stream` before reading out_h.  Calls
 * from several host threads are serialised by a library lock.  When the call
 * fails after some copies or kernels were queued, `stream` is still made to
 * wait for them before the error is returned: synchronise it before freeing
 * or reusing any buffer passed to the failed call.
 */
int halo_attn_host(const void* q_h, const void* k_h, const void* v_h, const void* rel_h_h, const void* rel_w_h,
                   void* out_h, void* q_d, void* k_d, void* v_d, void* rel_h_d, void* rel_w_d, void* out_d,
                   int N, int H, int W, int heads, int dim_head, int block, int halo, int stride, int dtype,
                   void* stream);

/*
 * halo_attn_masked -- the SASA-masked variant (section 2.2, the paragraph
 * after Figure 1: SASA uses the same blocking with halo = floor(k/2) and an
 * attention mask that emulates a k x k pixel-centred window).  Same
 * arguments and layouts as halo_attn plus `kernel` = k: each query keeps only
 * the window keys (Y, X) with |Y - y| <= k/2 and |X - x| <= k/2 (and inside
 * the image).  k must be odd with k/2 <= halo (HALO_ERR_KERNEL otherwise);
 * k = 2*halo + 1 is SASA's setting.  The relative tables are indexed as in
 * halo_attn.  Asynchronous on `stream`; allocates nothing.
 */
int halo_attn_masked(const void* q, const void* k, const void* v, const void* rel_h, const void* rel_w, void* out,
                     int N, int H, int W, int heads, int dim_head, int block, int halo, int stride, int kernel,
                     int dtype, void* stream);

/*
 * halo_attn_fused -- the same operation with the q, k, v projections done
 * inside the kernel (the blog page's HaloAttention module: q = x Wq^T and
 * [k | v] = x Wkv^T, bias-free linear maps of the input map x; HaloNet
 * appendix D: its speed-ups came from fusing around the attention op and
 * avoiding format changes).  x is read from HBM instead of stored q, k, v.
 *   x     : [N, H, W, c_in]        NHWC input map
 *   wq    : [heads*dim_head, c_in] query weights (a linear layer's [out, in])
 *   wkv   : [2*heads*dim_head, c_in] key rows first, then value rows
 *   rel_h, rel_w, out : as in halo_attn (out [N, H, W, heads*dim_head])
 * Every projection is accumulated in float32 and rounded to bf16 before the
 * attention, as a pipeline that stored q, k and v in bf16 would.  Supported:
 * bf16, block 8, stride 1, H/8 even, window 8..14 (halo 0..3), and
 * (dim_head, c_in) = (16, 64), (16, 128) or (32, 64); other shapes return
 * HALO_ERR_UNSUPPORTED (project with a GEMM and call halo_attn instead).
 * Pointers 16-byte aligned (HALO_ERR_ALIGN); out may not overlap an input
 * (HALO_ERR_ALIAS).  Asynchronous on `stream`; allocates nothing.
 */
int halo_attn_fused(const void* x, const void* wq, const void* wkv, const void* rel_h, const void* rel_w, void* out,
                    int N, int H, int W, int c_in, int heads, int dim_head, int block, int halo, int stride, int dtype,
                    void* stream);

/* Name of the kernel halo_attn_fused launches for this shape (e.g.
 * "halo_fused_tc<16,14,128>"), or "none" when it returns HALO_ERR_UNSUPPORTED
 * or rejects the shape.  Thread-local storage; never NULL. */
const char* halo_fused_kernel_name(int N, int H, int W, int c_in, int heads, int dim_head, int block, int halo,
                                   int stride, int dtype);

/*
 * halo_attn_bwd -- gradients of a loss L with respect to q, k, v, rel_h and
 * rel_w, given dout = dL/dout (the pages train this layer, section 2.2 and
 * Figure 3; the gradient is the chain rule through the operation above):
 *   with p the softmax weights of query i over its kept keys j,
 *   dz_ij = p_ij (dout_i . v_j - dout_i . out_i)
 *   dq_i  = s sum_j dz_ij (k_j + rel_h[a_ij] + rel_w[b_ij])
 *   dk_j  = s sum_i dz_ij q_i,   dv_j = sum_i p_ij dout_i  (over every window holding j)
 *   drel_h[a] = s sum over (image, head, query, key) with row index a of dz q, likewise drel_w
 *
 * Inputs (device, dtype `dtype`, 16-byte aligned): q, k, v, rel_h, rel_w as
 * for halo_attn; out = the forward's output for these inputs (same layout as
 * halo_attn's out; used for dout . out); dout = dL/dout, same layout.
 * Outputs (device, same dtype, 16-byte aligned, overlapping no input and no
 * other output): dq, dk, dv [N, H, W, heads*dim_head] (at stride 2 dq is zero
 * at pixels that are not queries), drel_h, drel_w [2w-1, dim_head].
 * `kernel`: 0 for halo_attn's operation, or the SASA mask size of
 * halo_attn_masked.
 * workspace: caller-owned device scratch of at least the size that
 * halo_attn_bwd_workspace_size reports, 256-byte aligned (HALO_ERR_WORKSPACE
 * otherwise); float32 accumulators, overwritten by the call.  The library
 * allocates nothing.  dim_head must be 8, 16, 32, 64 or 128, and one block's
 * window must fit the kernel's shared memory (HALO_ERR_UNSUPPORTED
 * otherwise).  Asynchronous on `stream`; the workspace must stay untouched
 * until the stream work is done.  Gradients are computed in float32 and
 * rounded to the dtype once.
 */
int halo_attn_bwd(const void* q, const void* k, const void* v, const void* rel_h, const void* rel_w,
                  const void* out, const void* dout, void* dq, void* dk, void* dv, void* drel_h, void* drel_w,
                  void* workspace, size_t workspace_bytes, int N, int H, int W, int heads, int dim_head, int block,
                  int halo, int stride, int kernel, int dtype, void* stream);

/* Name of the kernel halo_attn_bwd launches for these arguments (besides
 * zeroing the workspace and the finalize kernel), e.g. "halo_bwd_tc<16,14>"
 * or, at stride 2, "halo_bwd_tc<32,14,2>" (tensor cores: bf16, block 8,
 * dim_head 16 or 32, halo <= 3) or
 * "halo_bwd_simt<bf16,64>" (CUDA cores), or "none" when the shape is
 * rejected.  Thread-local storage as for halo_kernel_name; no device work. */
const char* halo_bwd_kernel_name(int N, int H, int W, int heads, int dim_head, int block, int halo, int stride,
                                 int kernel, int dtype);

/*
 * halo_attn_bwd_noalloc -- halo_attn_bwd for callers that cannot allocate
 * device memory when they run the backward.  The pages have no counterpart;
 * this is a convenience of this library.  Such callers are, for instance,
 * code whose device memory all belongs to a caching allocator (a cudaMalloc
 * of its own would fail once the allocator has reserved the free memory, or
 * would fragment it), and latency-critical paths where the device-wide
 * synchronisation that cudaMalloc and cudaFree can cause is not acceptable.
 *
 * Same arguments and results as halo_attn_bwd without workspace and
 * workspace_bytes: the float32 accumulators live in a static device array
 * of HALO_BWD_NOALLOC_MAX_WORKSPACE bytes (16 MiB) inside the library, which
 * every GPU that loads the library holds until the process exits.  Shapes
 * whose halo_attn_bwd_workspace_size exceeds that return
 * HALO_ERR_SCRATCH_LIMIT before any device work.  The call allocates
 * nothing (no cudaMalloc, cudaFree or allocating library routine); it
 * clears the part of the array it uses at the start of every call.
 *
 * The first call on a device looks up the array's device address on that
 * device (cudaGetSymbolAddress, with that device current) and keeps it; make
 * that first call before any stream capture.  Every call shares the one
 * array: calls whose work overlaps on the GPU (other streams, other host
 * threads, without ordering between them) race on it and give wrong
 * gradients.  Order such calls, or use halo_attn_bwd with a workspace each.
 */
#define HALO_BWD_NOALLOC_MAX_WORKSPACE (16u << 20)
int halo_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* rel_h, const void* rel_w,
                          const void* out, const void* dout, void* dq, void* dk, void* dv, void* drel_h,
                          void* drel_w, int N, int H, int W, int heads, int dim_head, int block, int halo,
                          int stride, int kernel, int dtype, void* stream);

/* Workspace bytes halo_attn_bwd needs for these arguments, in *bytes
 * (2 N H W heads dim_head + 2 (2w - 1) dim_head floats, each part rounded up
 * to 256 bytes).  Returns a halo_status; no device work. */
int halo_attn_bwd_workspace_size(int N, int H, int W, int heads, int dim_head, int block, int halo, int stride,
                                 int kernel, int dtype, size_t* bytes);

/* Which kernel halo_attn would launch for these arguments (halo_kernel_t),
 * or HALO_KERNEL_NONE when the shape is rejected.  No device work. */
int halo_kernel_for(int N, int H, int W, int heads, int dim_head, int block, int halo, int stride, int dtype);

/* Name of the kernel instantiation halo_attn would launch for these arguments,
 * e.g. "halo_fwd_tc2<16,14>" (template arguments: dim_head, window, and for
 * halo_fwd_tc the stride), or "none" when the shape is rejected.  The string
 * lives in thread-local storage of the library and stays valid until the next
 * halo_kernel_name call on the same thread; never NULL.  No device work. */
const char* halo_kernel_name(int N, int H, int W, int heads, int dim_head, int block, int halo, int stride,
                             int dtype);

/* As halo_kernel_name, for halo_attn_masked with mask size `kernel`
 * (e.g. "halo_fwd_tc4<16,14,masked>"); "none" when the shape is rejected. */
const char* halo_masked_kernel_name(int N, int H, int W, int heads, int dim_head, int block, int halo, int stride,
                                    int kernel, int dtype);

/* Static description of a status code; never NULL. */
const char* halo_strerror(int code);

/* Reads and clears the device error flag of the current device (HALO_OK or
 * HALO_ERR_TIMEOUT).  Synchronises the device. */
int halo_get_last_error(void);

/*
 * halo_debug_wait_timeout -- failure-detection self test.  Launches one tiny
 * kernel that waits on an mbarrier nobody arrives at, with a limit of
 * `limit_us` microseconds (1 .. 1000000); when the limit runs out the kernel
 * records HALO_ERR_TIMEOUT in a flag of its own and returns normally.
 * Returns that flag's value (it synchronises `stream`), so a working timeout
 * path returns HALO_ERR_TIMEOUT.  It neither reads nor clears the flag that
 * halo_get_last_error reports, so a timeout recorded by an earlier halo_attn
 * stays there.  Touches no caller memory.
 */
int halo_debug_wait_timeout(int limit_us, void* stream);

/* Library version: major*10000 + minor*100 + patch. */
int halo_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HALO_H_ */
