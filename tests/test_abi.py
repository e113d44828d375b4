"""The C ABI: libhalo.so loads without a GPU, exports every entry point that
include/halo.h declares, and rejects invalid arguments before touching the
device (no kernel is launched by these tests)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "halo.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(halo_\w+)\s*\(", src, flags=re.M)))


def _lib():
    from blocked_local_self_b200 import _native
    return _native.lib()


def test_header_declares_the_boundary():
    names = _declared_functions()
    for expected in ("halo_attn", "halo_attn_host", "halo_kernel_for", "halo_kernel_name", "halo_strerror",
                     "halo_get_last_error",
                     "halo_debug_wait_timeout", "halo_version"):
        assert expected in names


def test_library_exports_every_declared_symbol():
    lib = _lib()
    for name in _declared_functions():
        assert hasattr(lib, name), f"libhalo.so does not export {name}"


def test_binding_mirrors_header():
    from blocked_local_self_b200 import _native
    assert sorted(_native.SIGNATURES) == _declared_functions()


def test_status_codes_match_header():
    from blocked_local_self_b200 import _native
    src = open(HEADER).read()
    for name, val in re.findall(r"(HALO_(?:OK|ERR_\w+))\s*=\s*(-?\d+)", src):
        assert getattr(_native, name) == int(val), name


def test_strerror_covers_codes():
    lib = _lib()
    for code in range(0, -15, -1):
        text = lib.halo_strerror(code).decode()
        assert text and text != "unknown status code"
    assert lib.halo_strerror(-99).decode() == "unknown status code"


def test_version():
    assert _lib().halo_version() >= 100


ARGS = dict(N=1, H=16, W=16, heads=2, d=16, block=8, halo=3, stride=1, dtype=1)


def _call(ptrs=(16,) * 6, **over):
    a = dict(ARGS, **over)
    return _lib().halo_attn(*ptrs, a["N"], a["H"], a["W"], a["heads"], a["d"], a["block"], a["halo"],
                            a["stride"], a["dtype"], None)


@pytest.mark.parametrize("over,code", [
    (dict(dtype=7), -9),
    (dict(N=0), -2), (dict(H=-8), -2), (dict(heads=0), -2), (dict(d=0), -2), (dict(block=0), -2),
    (dict(halo=-1), -2),
    (dict(stride=3), -4),
    (dict(H=12), -3), (dict(W=20), -3), (dict(block=3, stride=2, H=9, W=9), -3),
    (dict(heads=1, d=4), -5),
])
def test_shape_checks(over, code):
    assert _call(**over) == code


def test_pointer_checks():
    assert _call(ptrs=(16, 16, 0, 16, 16, 16)) == -1
    assert _call(ptrs=(16, 16, 24, 16, 16, 4096)) == -5
    # out overlapping q: q at 1<<20, out 256 bytes later
    assert _call(ptrs=(1 << 20, 1 << 22, 1 << 23, 1 << 24, 1 << 25, (1 << 20) + 256)) == -10


def test_kernel_selection_is_host_only():
    lib = _lib()
    # the stage-1 HaloNet layer goes to the tensor-core kernel
    assert lib.halo_kernel_for(32, 64, 64, 8, 16, 8, 3, 1, 1) == 2
    assert lib.halo_kernel_for(64, 32, 32, 8, 64, 8, 3, 1, 1) == 2
    assert lib.halo_kernel_for(64, 64, 64, 8, 32, 8, 3, 2, 1) == 2
    # float32 goes to the CUDA-core kernel, invalid shapes to none
    assert lib.halo_kernel_for(1, 16, 16, 2, 32, 4, 1, 1, 0) == 1
    assert lib.halo_kernel_for(1, 16, 16, 2, 32, 5, 1, 1, 0) == 0
    # 16x16 blocks with a 4-pixel halo go to the block-16 tensor-core kernel
    assert lib.halo_kernel_for(16, 128, 128, 8, 32, 16, 4, 1, 1) == 2


def test_kernel_names():
    lib = _lib()
    name = lambda *a: lib.halo_kernel_name(*a).decode()
    assert name(32, 64, 64, 8, 16, 8, 3, 1, 1) == "halo_fwd_tc4<16,14>"  # even number of block rows
    assert name(2, 32, 32, 8, 16, 8, 1, 1, 1) == "halo_fwd_tc4<16,10>"
    assert name(2, 32, 32, 8, 32, 8, 3, 1, 1) == "halo_fwd_tc4<32,14>"
    assert name(2, 24, 32, 8, 16, 8, 3, 1, 1) == "halo_fwd_tc2<16,14>"  # odd: head pairs
    assert name(2, 40, 32, 8, 32, 8, 2, 1, 1) == "halo_fwd_tc2<32,12>"
    assert name(64, 32, 32, 8, 64, 8, 3, 1, 1) == "halo_fwd_tc4<64,14>"
    assert name(64, 24, 32, 8, 64, 8, 3, 1, 1) == "halo_fwd_tc<64,14,1,1>"  # odd number of block rows
    assert name(2, 16, 24, 3, 16, 8, 3, 1, 1) == "halo_fwd_tc4<16,14>"   # odd head count, even block rows
    assert name(2, 24, 24, 3, 16, 8, 3, 1, 1) == "halo_fwd_tc<16,14,1,1>"   # odd head count, odd block rows
    assert name(2, 32, 48, 3, 16, 16, 2, 1, 1) == "halo_fwd_tc3<16,20,16>"
    assert name(64, 64, 64, 8, 32, 8, 3, 2, 1) == "halo_fwd_tc<32,14,2,4>"  # four heads per 64-row tile
    assert name(64, 64, 64, 6, 32, 8, 3, 2, 1) == "halo_fwd_tc<32,14,2,2>"  # six heads: pairs
    assert name(16, 128, 128, 8, 32, 16, 4, 1, 1) == "halo_fwd_tc3<32,24,16>"
    assert name(1, 16, 16, 2, 32, 4, 1, 1, 0) == "halo_fwd_win<float,32>"   # window staged in shared memory
    assert name(1, 16, 16, 2, 40, 4, 1, 1, 0) == "halo_fwd_simt<float,64>"  # dim_head the staged kernel lacks
    assert name(2, 32, 32, 4, 40, 16, 4, 1, 1) == "halo_fwd_simt<bf16,64>"
    assert name(1, 16, 16, 2, 32, 5, 1, 1, 0) == "none"


def test_bwd_kernel_names():
    """The backward's kernel choice (host-only): the tensor-core kernel for
    bf16 8x8 blocks with d 16 or 32 at stride 1 and 2 (the stride-2 form named
    with its stride), the CUDA-core kernel for every other shape."""
    lib = _lib()
    name = lambda *a: lib.halo_bwd_kernel_name(*a).decode()
    assert name(32, 64, 64, 8, 16, 8, 3, 1, 0, 1) == "halo_bwd_tc<16,14>"
    assert name(2, 32, 32, 4, 32, 8, 2, 1, 0, 1) == "halo_bwd_tc<32,12>"
    assert name(64, 64, 64, 8, 32, 8, 3, 2, 0, 1) == "halo_bwd_tc<32,14,2>"
    assert name(2, 32, 32, 4, 16, 8, 0, 2, 0, 1) == "halo_bwd_tc<16,8,2>"
    assert name(1, 16, 16, 2, 16, 8, 3, 2, 5, 1) == "halo_bwd_tc<16,14,2>"   # SASA mask
    assert name(64, 32, 32, 8, 64, 8, 3, 1, 0, 1) == "halo_bwd_simt<bf16,64>"
    assert name(1, 16, 16, 2, 32, 8, 3, 2, 0, 0) == "halo_bwd_simt<float,32>"
    assert name(1, 32, 32, 2, 32, 16, 4, 1, 0, 1) == "halo_bwd_simt<bf16,32>"  # block 16
    assert name(1, 16, 16, 2, 32, 5, 1, 1, 0, 1) == "none"


def test_fused_kernel_selection():
    lib = _lib()
    name = lambda *a: lib.halo_fused_kernel_name(*a).decode()
    # (N, H, W, c_in, heads, d, block, halo, stride, dtype)
    assert name(32, 64, 64, 128, 8, 16, 8, 3, 1, 1) == "halo_fused_tc<16,14,128>"
    assert name(2, 16, 16, 64, 2, 16, 8, 2, 1, 1) == "halo_fused_tc<16,12,64>"
    assert name(2, 32, 32, 64, 4, 32, 8, 0, 1, 1) == "halo_fused_tc<32,8,64>"
    assert name(2, 32, 32, 128, 4, 32, 8, 3, 1, 1) == "none"   # d 32 with c_in 128: no room in shared memory
    assert name(2, 24, 32, 128, 8, 16, 8, 3, 1, 1) == "none"   # odd number of block rows
    assert name(2, 32, 32, 96, 8, 16, 8, 3, 1, 1) == "none"    # c_in 96
    assert name(2, 32, 32, 128, 8, 16, 8, 3, 2, 1) == "none"   # stride 2
    assert name(2, 32, 32, 128, 8, 16, 8, 3, 1, 0) == "none"   # float32
    assert name(2, 32, 32, 128, 8, 16, 16, 3, 1, 1) == "none"  # block 16


def _fused(ptrs=(16,) * 6, **over):
    a = dict(dict(ARGS, c_in=128), **over)
    return _lib().halo_attn_fused(*ptrs, a["N"], a["H"], a["W"], a["c_in"], a["heads"], a["d"], a["block"],
                                  a["halo"], a["stride"], a["dtype"], None)


def test_fused_entry_checks_on_the_host():
    assert _fused(N=0) == -2
    assert _fused(c_in=0) == -2
    assert _fused(H=12) == -3
    assert _fused(ptrs=(16, 0, 16, 16, 16, 16)) == -1
    assert _fused(ptrs=(16, 24, 16, 16, 16, 4096)) == -5
    assert _fused(c_in=4) == -5                     # x rows of 8 bytes
    # out overlapping the weights
    assert _fused(ptrs=(1 << 20, 1 << 22, 1 << 23, 1 << 24, 1 << 25, (1 << 22) + 256)) == -10
    # valid arguments, shape without a fused kernel: refused before any device call
    assert _fused(ptrs=(1 << 20, 1 << 22, 1 << 23, 1 << 24, 1 << 25, 1 << 26), c_in=96) == -6
    assert _fused(ptrs=(1 << 20, 1 << 22, 1 << 23, 1 << 24, 1 << 25, 1 << 26), stride=2) == -6


def test_host_entry_checks_before_any_copy():
    lib = _lib()
    a = ARGS
    rc = lib.halo_attn_host(*([16] * 5 + [None]), *([16] * 6), a["N"], a["H"], a["W"], a["heads"], a["d"],
                            a["block"], a["halo"], a["stride"], a["dtype"], None)
    assert rc == -1


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    from blocked_local_self_b200 import _native
    monkeypatch.setattr(_native, "LIB_PATH", str(tmp_path / "libhalo.so"))
    monkeypatch.setattr(_native, "_lib", None)
    with pytest.raises(ImportError):
        _native.lib()
