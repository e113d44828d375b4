"""blocked_local_self_b200 -- HaloNet blocked local self-attention with
haloing on NVIDIA B200 (sm_100a).

The computation runs entirely in ``libhalo.so`` (hand-written CUDA, C ABI in
``include/halo.h``).  This module only marshals torch tensors (device memory
and streams) into that ABI.

    out = attn(q, k, v, rel_h, rel_w, block=8, halo=3, stride=1)

q, k, v: NHWC ``[N, H, W, heads*dim_head]`` CUDA tensors (bf16 or float32),
rel_h, rel_w: ``[2*(block+2*halo)-1, dim_head]`` of the same dtype.
Returns ``[N, H/stride, W/stride, heads*dim_head]``.
"""
from __future__ import annotations

import torch

from . import _native
from ._native import HaloError, HALO_BF16, HALO_F32

__all__ = ["attn", "attn_masked", "attn_bwd", "bwd_workspace_size", "attn_host", "kernel_for", "kernel_name",
           "masked_kernel_name", "bwd_kernel_name", "get_last_error", "debug_wait_timeout", "version", "HaloError", "load"]


def load():
    """Load libhalo.so (raises ImportError when it has not been built)."""
    return _native.lib()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return HALO_BF16
    if t.dtype == torch.float32:
        return HALO_F32
    raise TypeError(f"unsupported dtype {t.dtype}; expected bfloat16 or float32")


def _sizes(q: torch.Tensor, rel_h: torch.Tensor, heads: int | None):
    if q.dim() != 4 or rel_h.dim() != 2:
        raise ValueError("q must be [N, H, W, C] and rel_h [2w-1, dim_head]")
    N, H, W, C = q.shape
    d = rel_h.shape[1]
    if heads is None:
        if C % d:
            raise ValueError(f"channels {C} not a multiple of dim_head {d}")
        heads = C // d
    return N, H, W, heads, d


def _stream_ptr(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, rel_h: torch.Tensor, rel_w: torch.Tensor,
         block: int, halo: int, stride: int = 1, heads: int | None = None, out: torch.Tensor | None = None,
         stream=None) -> torch.Tensor:
    """Blocked local self-attention with haloing on device tensors (asynchronous
    on ``stream``, default: torch's current stream)."""
    tensors = (q, k, v, rel_h, rel_w)
    for t in tensors:
        if not t.is_cuda:
            raise ValueError("attn expects CUDA tensors; use attn_host for host buffers")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    N, H, W, heads, d = _sizes(q, rel_h, heads)
    code = _dtype_code(q)
    if out is None:
        out = torch.empty((N, H // stride, W // stride, heads * d), dtype=q.dtype, device=q.device)
    rc = _native.lib().halo_attn(q.data_ptr(), k.data_ptr(), v.data_ptr(), rel_h.data_ptr(), rel_w.data_ptr(),
                                 out.data_ptr(), N, H, W, heads, d, block, halo, stride, code, _stream_ptr(stream))
    if rc != 0:
        raise HaloError(rc)
    return out


def attn_masked(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, rel_h: torch.Tensor, rel_w: torch.Tensor,
                block: int, halo: int, kernel: int, stride: int = 1, heads: int | None = None,
                out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """SASA-masked variant: each query keeps only the ``kernel`` x ``kernel``
    keys centred on it (``halo_attn_masked``)."""
    for t in (q, k, v, rel_h, rel_w):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("attn_masked expects contiguous CUDA tensors")
    N, H, W, heads, d = _sizes(q, rel_h, heads)
    if out is None:
        out = torch.empty((N, H // stride, W // stride, heads * d), dtype=q.dtype, device=q.device)
    rc = _native.lib().halo_attn_masked(q.data_ptr(), k.data_ptr(), v.data_ptr(), rel_h.data_ptr(),
                                        rel_w.data_ptr(), out.data_ptr(), N, H, W, heads, d, block, halo, stride,
                                        kernel, _dtype_code(q), _stream_ptr(stream))
    if rc != 0:
        raise HaloError(rc, "halo_attn_masked")
    return out


def attn_fused(x: torch.Tensor, wq: torch.Tensor, wkv: torch.Tensor, rel_h: torch.Tensor, rel_w: torch.Tensor,
               heads: int, block: int, halo: int, stride: int = 1, out: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """The operation with the q, k, v projections inside the kernel
    (``halo_attn_fused``): ``x`` is the NHWC input map [N, H, W, c_in], ``wq``
    [heads*d, c_in] and ``wkv`` [2*heads*d, c_in] are bias-free linear layers'
    weights ([out, in]; key rows, then value rows)."""
    for t in (x, wq, wkv, rel_h, rel_w):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("attn_fused expects contiguous CUDA tensors")
    if x.dim() != 4 or wq.dim() != 2 or wkv.dim() != 2:
        raise ValueError("x must be [N, H, W, c_in], wq [heads*d, c_in], wkv [2*heads*d, c_in]")
    N, H, W, c_in = x.shape
    d = rel_h.shape[-1]
    if wq.shape != (heads * d, c_in) or wkv.shape != (2 * heads * d, c_in):
        raise ValueError("weight shapes do not match heads, dim_head and c_in")
    if out is None:
        out = torch.empty((N, H // stride, W // stride, heads * d), dtype=x.dtype, device=x.device)
    rc = _native.lib().halo_attn_fused(x.data_ptr(), wq.data_ptr(), wkv.data_ptr(), rel_h.data_ptr(),
                                       rel_w.data_ptr(), out.data_ptr(), N, H, W, c_in, heads, d, block, halo,
                                       stride, _dtype_code(x), _stream_ptr(stream))
    if rc != 0:
        raise HaloError(rc, "halo_attn_fused")
    return out


def bwd_workspace_size(N: int, H: int, W: int, heads: int, dim_head: int, block: int, halo: int, stride: int,
                       kernel: int, dtype: torch.dtype) -> int:
    """Bytes of device workspace ``attn_bwd`` needs (``halo_attn_bwd_workspace_size``)."""
    import ctypes
    nb = ctypes.c_size_t(0)
    code = HALO_BF16 if dtype == torch.bfloat16 else HALO_F32
    rc = _native.lib().halo_attn_bwd_workspace_size(N, H, W, heads, dim_head, block, halo, stride, kernel, code,
                                                    ctypes.byref(nb))
    if rc != 0:
        raise HaloError(rc, "halo_attn_bwd_workspace_size")
    return int(nb.value)


def attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, rel_h: torch.Tensor, rel_w: torch.Tensor,
             out: torch.Tensor, dout: torch.Tensor, block: int, halo: int, stride: int = 1, kernel: int = 0,
             heads: int | None = None, grads: tuple | None = None, workspace: torch.Tensor | None = None,
             stream=None):
    """Gradients (dq, dk, dv, drel_h, drel_w) of ``sum(out * dout)``
    (``halo_attn_bwd``).  ``out`` is the forward's output for these inputs.
    ``grads`` may pass preallocated outputs and ``workspace`` a uint8 CUDA
    tensor of at least ``bwd_workspace_size`` bytes."""
    for t in (q, k, v, rel_h, rel_w, out, dout):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("attn_bwd expects contiguous CUDA tensors")
    N, H, W, heads, d = _sizes(q, rel_h, heads)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(rel_h),
                 torch.empty_like(rel_w))
    nbytes = bwd_workspace_size(N, H, W, heads, d, block, halo, stride, kernel, q.dtype)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    rc = _native.lib().halo_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), rel_h.data_ptr(), rel_w.data_ptr(),
                                     out.data_ptr(), dout.data_ptr(), *[g_.data_ptr() for g_ in grads],
                                     workspace.data_ptr(), workspace.numel() * workspace.element_size(), N, H, W,
                                     heads, d, block, halo, stride, kernel, _dtype_code(q), _stream_ptr(stream))
    if rc != 0:
        raise HaloError(rc, "halo_attn_bwd")
    return grads


def attn_host(q_h: torch.Tensor, k_h: torch.Tensor, v_h: torch.Tensor, rel_h_h: torch.Tensor,
              rel_w_h: torch.Tensor, out_h: torch.Tensor, staging: dict, block: int, halo: int, stride: int = 1,
              heads: int | None = None, stream=None) -> torch.Tensor:
    """End-to-end form on host tensors: copies in, kernel, copy out, all queued
    on ``stream`` by libhalo.  ``staging`` holds caller-allocated device tensors
    ``q, k, v, rel_h, rel_w, out`` of matching sizes.  Synchronise the stream
    before reading ``out_h``."""
    N, H, W, heads, d = _sizes(q_h, rel_h_h, heads)
    code = _dtype_code(q_h)
    s = staging
    rc = _native.lib().halo_attn_host(
        q_h.data_ptr(), k_h.data_ptr(), v_h.data_ptr(), rel_h_h.data_ptr(), rel_w_h.data_ptr(), out_h.data_ptr(),
        s["q"].data_ptr(), s["k"].data_ptr(), s["v"].data_ptr(), s["rel_h"].data_ptr(), s["rel_w"].data_ptr(),
        s["out"].data_ptr(), N, H, W, heads, d, block, halo, stride, code, _stream_ptr(stream))
    if rc != 0:
        raise HaloError(rc, "halo_attn_host")
    return out_h


def kernel_for(N: int, H: int, W: int, heads: int, dim_head: int, block: int, halo: int, stride: int,
               dtype: torch.dtype) -> str:
    """Name of the kernel ``attn`` launches for a shape: "tc_bf16", "simt_f32" or "none"."""
    code = HALO_BF16 if dtype == torch.bfloat16 else HALO_F32
    k = _native.lib().halo_kernel_for(N, H, W, heads, dim_head, block, halo, stride, code)
    return {0: "none", 1: "simt_f32", 2: "tc_bf16"}[k]


def kernel_name(N: int, H: int, W: int, heads: int, dim_head: int, block: int, halo: int, stride: int,
                dtype: torch.dtype) -> str:
    """Instantiation ``attn`` launches for a shape, e.g. "halo_fwd_tc2<16,14>", or "none"."""
    code = HALO_BF16 if dtype == torch.bfloat16 else HALO_F32
    return _native.lib().halo_kernel_name(N, H, W, heads, dim_head, block, halo, stride, code).decode()


def masked_kernel_name(N: int, H: int, W: int, heads: int, dim_head: int, block: int, halo: int, stride: int,
                       kernel: int, dtype: torch.dtype) -> str:
    """Instantiation ``attn_masked`` launches for a shape, or "none"."""
    code = HALO_BF16 if dtype == torch.bfloat16 else HALO_F32
    return _native.lib().halo_masked_kernel_name(N, H, W, heads, dim_head, block, halo, stride, kernel,
                                                 code).decode()


def fused_kernel_name(N: int, H: int, W: int, c_in: int, heads: int, dim_head: int, block: int, halo: int,
                      stride: int, dtype: torch.dtype) -> str:
    """Kernel ``attn_fused`` launches for a shape, or "none"."""
    code = HALO_BF16 if dtype == torch.bfloat16 else HALO_F32
    return _native.lib().halo_fused_kernel_name(N, H, W, c_in, heads, dim_head, block, halo, stride,
                                                code).decode()


def bwd_kernel_name(N: int, H: int, W: int, heads: int, dim_head: int, block: int, halo: int, stride: int,
                    kernel: int, dtype: torch.dtype) -> str:
    """Kernel ``attn_bwd`` launches for a shape, or "none"."""
    code = HALO_BF16 if dtype == torch.bfloat16 else HALO_F32
    return _native.lib().halo_bwd_kernel_name(N, H, W, heads, dim_head, block, halo, stride, kernel,
                                              code).decode()


def get_last_error() -> int:
    return _native.lib().halo_get_last_error()


def debug_wait_timeout(limit_us: int, stream=None) -> int:
    return _native.lib().halo_debug_wait_timeout(limit_us, _stream_ptr(stream))


def version() -> int:
    return _native.lib().halo_version()
