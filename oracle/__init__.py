"""CPU oracle for HaloNet blocked local self-attention (test infrastructure).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The CUDA path
(``blocked_local_self_b200``) never imports this package and shares no code
with it; the two meet only through the seeded inputs of ``workloads``.

The arithmetic lives in ``halo_oracle.c`` (plain C, double precision, one
loop nest per output pixel and head, see the header comment there for the
passages of the HaloNet pages it follows).  This module compiles it with gcc
and calls it through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "halo_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

DTYPE_F32 = 0
DTYPE_BF16 = 1

_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to the source (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        vp, ip, dp = ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(ctypes.c_double)
        lib.halo_oracle_f64.argtypes = [vp] * 5 + [dp] + [ip] * 10
        lib.halo_oracle_f64.restype = ip
        lib.halo_oracle_samples_f64.argtypes = [vp] * 5 + [ctypes.POINTER(ctypes.c_int), ip, dp] + [ip] * 10
        lib.halo_oracle_samples_f64.restype = ip
        lib.halo_oracle_masked_f64.argtypes = [vp] * 5 + [dp] + [ip] * 11
        lib.halo_oracle_masked_f64.restype = ip
        lib.halo_oracle_bwd_f64.argtypes = [vp] * 6 + [dp] * 5 + [ip] * 11
        lib.halo_oracle_bwd_f64.restype = ip
        lib.halo_oracle_fused_f64.argtypes = [vp] * 5 + [dp] + [ip] * 11
        lib.halo_oracle_fused_f64.restype = ip
        lib.halo_oracle_max_threads.argtypes = []
        lib.halo_oracle_max_threads.restype = ip
        _lib = lib
    return _lib


def _as_host_array(t):
    """Return (numpy array holding the raw stored values, dtype code)."""
    import torch

    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16), DTYPE_BF16
        if t.dtype == torch.float32:
            return t.numpy(), DTYPE_F32
        raise TypeError(f"unsupported dtype {t.dtype}")
    a = np.ascontiguousarray(t)
    if a.dtype == np.float32:
        return a, DTYPE_F32
    if a.dtype == np.uint16:
        return a, DTYPE_BF16
    raise TypeError(f"unsupported dtype {a.dtype}")


def _prepare(q, k, v, rel_h, rel_w):
    arrs = [_as_host_array(t) for t in (q, k, v, rel_h, rel_w)]
    codes = {c for _, c in arrs}
    if len(codes) != 1:
        raise TypeError("q, k, v, rel_h, rel_w must share one dtype")
    return [a for a, _ in arrs], codes.pop()


def max_threads() -> int:
    return int(_load().halo_oracle_max_threads())


def halo_attention(q, k, v, rel_h, rel_w, block: int, halo: int, stride: int = 1,
                   heads: int | None = None, threads: int = 0) -> np.ndarray:
    """Full oracle output as float64 ``[N, H/stride, W/stride, C]``.

    q, k, v: NHWC ``[N, H, W, heads*d]``; rel_h, rel_w: ``[2(b+2h)-1, d]``.
    """
    lib = _load()
    (qa, ka, va, rha, rwa), code = _prepare(q, k, v, rel_h, rel_w)
    N, H, W, C = qa.shape
    d = rha.shape[1]
    if heads is None:
        heads = C // d
    out = np.empty((N, H // stride, W // stride, C), dtype=np.float64)
    rc = lib.halo_oracle_f64(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, rha.ctypes.data, rwa.ctypes.data,
                             out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                             N, H, W, heads, d, block, halo, stride, code, threads)
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")
    return out


def halo_attention_samples(q, k, v, rel_h, rel_w, samples, block: int, halo: int, stride: int = 1,
                           heads: int | None = None, threads: int = 0) -> np.ndarray:
    """Oracle output at sampled pixels: ``samples`` is an int array [S, 3] of
    (n, oy, ox); returns float64 ``[S, C]``."""
    lib = _load()
    (qa, ka, va, rha, rwa), code = _prepare(q, k, v, rel_h, rel_w)
    N, H, W, C = qa.shape
    d = rha.shape[1]
    if heads is None:
        heads = C // d
    smp = np.ascontiguousarray(np.asarray(samples, dtype=np.int32).reshape(-1, 3))
    out = np.empty((smp.shape[0], C), dtype=np.float64)
    rc = lib.halo_oracle_samples_f64(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, rha.ctypes.data,
                                     rwa.ctypes.data, smp.ctypes.data_as(ctypes.POINTER(ctypes.c_int)),
                                     smp.shape[0], out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                                     N, H, W, heads, d, block, halo, stride, code, threads)
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")
    return out


def halo_attention_masked(q, k, v, rel_h, rel_w, block: int, halo: int, kernel: int, stride: int = 1,
                          heads: int | None = None, threads: int = 0) -> np.ndarray:
    """SASA-masked variant: each query keeps only the ``kernel`` x ``kernel``
    keys centred on it (``kernel`` odd, ``kernel // 2 <= halo``).  Float64
    ``[N, H/stride, W/stride, C]``."""
    lib = _load()
    (qa, ka, va, rha, rwa), code = _prepare(q, k, v, rel_h, rel_w)
    N, H, W, C = qa.shape
    d = rha.shape[1]
    if heads is None:
        heads = C // d
    out = np.empty((N, H // stride, W // stride, C), dtype=np.float64)
    rc = lib.halo_oracle_masked_f64(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, rha.ctypes.data,
                                    rwa.ctypes.data, out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                                    N, H, W, heads, d, block, halo, stride, kernel, code, threads)
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")
    return out


def halo_attention_bwd(q, k, v, rel_h, rel_w, dout, block: int, halo: int, stride: int = 1, kernel: int = 0,
                       heads: int | None = None, threads: int = 0):
    """Gradients of ``sum(out * dout)`` with respect to q, k, v, rel_h, rel_w
    (float64 arrays ``dq, dk, dv`` of q's shape and ``drel_h, drel_w`` of the
    tables' shape).  ``dout``: ``[N, H/stride, W/stride, C]`` in the inputs'
    dtype.  ``kernel`` > 0 applies the SASA mask as in
    ``halo_attention_masked``."""
    lib = _load()
    (qa, ka, va, rha, rwa, da), code = _prepare_n(q, k, v, rel_h, rel_w, dout)
    N, H, W, C = qa.shape
    d = rha.shape[1]
    if heads is None:
        heads = C // d
    grads = [np.empty(qa.shape, dtype=np.float64) for _ in range(3)]
    grads += [np.empty(rha.shape, dtype=np.float64) for _ in range(2)]
    dptr = [g.ctypes.data_as(ctypes.POINTER(ctypes.c_double)) for g in grads]
    rc = lib.halo_oracle_bwd_f64(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, rha.ctypes.data, rwa.ctypes.data,
                                 da.ctypes.data, *dptr, N, H, W, heads, d, block, halo, stride, kernel, code,
                                 threads)
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")
    return tuple(grads)


def _prepare_n(*tensors):
    arrs = [_as_host_array(t) for t in tensors]
    codes = {c for _, c in arrs}
    if len(codes) != 1:
        raise TypeError("all tensors must share one dtype")
    return [a for a, _ in arrs], codes.pop()


def halo_attention_fused(x, wq, wkv, rel_h, rel_w, block: int, halo: int, heads: int, stride: int = 1,
                         threads: int = 0) -> np.ndarray:
    """Fused projections: q = x wq^T, [k | v] = x wkv^T per pixel (exact, each
    rounded to the inputs' dtype), then the operation.  x: ``[N, H, W, c_in]``;
    wq: ``[heads*d, c_in]``; wkv: ``[2*heads*d, c_in]``.  Float64
    ``[N, H/stride, W/stride, heads*d]``."""
    lib = _load()
    (xa, qa, ka, rha, rwa), code = _prepare_n(x, wq, wkv, rel_h, rel_w)
    N, H, W, c_in = xa.shape
    d = rha.shape[1]
    C = qa.shape[0]
    out = np.empty((N, H // stride, W // stride, C), dtype=np.float64)
    rc = lib.halo_oracle_fused_f64(xa.ctypes.data, qa.ctypes.data, ka.ctypes.data, rha.ctypes.data,
                                   rwa.ctypes.data, out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                                   N, H, W, c_in, heads, d, block, halo, stride, code, threads)
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")
    return out
