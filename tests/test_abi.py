"""CPU: libhstu_attn.so builds for sm_100a, loads, and exports every function include/hstu_attn.h
declares; host-side argument validation answers synchronously without touching a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hstu_attn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hstu_(?:attn|layer|layers)_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    assert declared_functions() == sorted(["hstu_attn_fwd", "hstu_attn_fwd_cached", "hstu_attn_fwd_rab",
                                           "hstu_attn_plan_bytes",
                                           "hstu_attn_plan", "hstu_attn_fwd_planned", "hstu_attn_fwd_noalloc",
                                           "hstu_attn_get_error", "hstu_attn_status_string",
                                           "hstu_attn_selfcheck_wait_timeout", "hstu_attn_gemm_bf16",
                                           "hstu_attn_bwd", "hstu_attn_bwd_workspace_limit", "hstu_attn_partition",
                                           "hstu_layer_workspace_bytes",
                                           "hstu_layer_fwd", "hstu_layers_fwd", "hstu_attn_selfcheck_fwd_timeout"])


def test_library_exports_every_declared_symbol(cuda_lib):
    from hstu_pointwise_attention_jagged_b200 import binding
    for name in declared_functions():
        assert hasattr(cuda_lib, name), name
    assert sorted(binding.EXPORTS) == declared_functions()
    # the exported names are plain C symbols
    out = os.popen("nm -D --defined-only %s" % binding.library_path()).read()
    for name in declared_functions():
        assert re.search(r"\sT %s$" % name, out, re.M), name


def test_status_strings(cuda_lib):
    names = [cuda_lib.hstu_attn_status_string(i).decode() for i in range(6)]
    assert names == ["HSTU_OK", "HSTU_ERR_INVALID_ARGUMENT", "HSTU_ERR_UNSUPPORTED", "HSTU_ERR_CUDA",
                     "HSTU_ERR_BAD_OFFSETS", "HSTU_ERR_TIMEOUT"]


def test_plan_bytes(cuda_lib):
    """16-byte header, B query-row starts and B+1 block starts (each padded to 16 bytes), 16 bytes
    per possible item."""
    assert cuda_lib.hstu_attn_plan_bytes(8, 4, 32768) == 16 + 32 + 48 + 16 * 4 * (32768 // 128 + 8)
    assert cuda_lib.hstu_attn_plan_bytes(3, 1, 10) == 16 + 16 + 16 + 16 * 3
    assert cuda_lib.hstu_attn_plan_bytes(-1, 4, 10) == 0


def _fwd(lib, **kw):
    args = dict(q=1 << 12, k=1 << 12, v=1 << 12, off=1 << 12, nt=None, B=1, H=2, d=128, total=16,
                msl=16, alpha=1.0, N=16.0, out=1 << 20, stream=None)
    args.update(kw)
    vp = ctypes.c_void_p
    return lib.hstu_attn_fwd(vp(args["q"]), vp(args["k"]), vp(args["v"]), vp(args["off"]), vp(args["nt"]),
                             args["B"], args["H"], args["d"], args["total"], args["msl"], args["alpha"], args["N"],
                             vp(args["out"]), vp(args["stream"]))


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(off=None), 1), (dict(out=None), 1), (dict(B=-1), 1), (dict(H=0), 1),
    (dict(N=0.0), 1), (dict(N=float("nan")), 1), (dict(alpha=float("inf")), 1), (dict(total=-5), 1),
    (dict(d=48), 2), (dict(d=256), 2), (dict(q=(1 << 12) + 8), 2), (dict(out=1 << 12), 1),
])
def test_host_validation(cuda_lib, kw, status):
    """Rejected before any CUDA call: no GPU is needed to see these statuses."""
    assert _fwd(cuda_lib, **kw) == status


def test_host_validation_cached_and_planned(cuda_lib):
    vp = ctypes.c_void_p
    # total_q > total_kv is impossible
    st = cuda_lib.hstu_attn_fwd_cached(vp(4096), vp(4096), vp(4096), vp(4096), None, None, 1, 1, 64, 10, 11, 10,
                                       1.0, 1.0, vp(1 << 20), None)
    assert st == 1
    # a plan buffer smaller than hstu_attn_plan_bytes
    st = cuda_lib.hstu_attn_plan(vp(4096), None, None, 2, 1, 10, 10, 10, vp(1 << 20), 16, None)
    assert st == 1
    # fwd_planned without a plan
    st = cuda_lib.hstu_attn_fwd_planned(vp(4096), vp(4096), vp(4096), vp(4096), None, None, 1, 1, 64, 10, 10,
                                        1.0, 1.0, None, vp(1 << 20), None)
    assert st == 1
    # the bias variant needs a table of 1 .. 2^24 entries per head
    cuda_lib.hstu_attn_fwd_rab.argtypes = [vp] * 7 + [ctypes.c_int32] * 7 + [ctypes.c_float] * 2 + [vp, vp]
    assert cuda_lib.hstu_attn_fwd_rab(vp(4096), vp(4096), vp(4096), vp(4096), None, None, None, 16, 1, 1, 64, 10, 10,
                                      10, 1.0, 1.0, vp(1 << 20), None) == 1
    assert cuda_lib.hstu_attn_fwd_rab(vp(4096), vp(4096), vp(4096), vp(4096), None, None, vp(4096), 0, 1, 1, 64, 10,
                                      10, 10, 1.0, 1.0, vp(1 << 20), None) == 1
    # the GEMM: K and N multiples of 8, aligned pointers, no overlap of C with A or W
    g = cuda_lib.hstu_attn_gemm_bf16
    g.argtypes = [vp, vp, vp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, vp]
    assert g(vp(4096), vp(1 << 22), vp(1 << 24), 16, 16, 12, None) == 2      # K % 8
    assert g(vp(4096), vp(1 << 22), vp(1 << 24), 16, 12, 16, None) == 2      # N % 8
    assert g(vp(4100), vp(1 << 22), vp(1 << 24), 16, 16, 16, None) == 2      # misaligned A
    assert g(vp(4096), vp(1 << 22), vp(4096 + 64), 16, 16, 16, None) == 1    # C overlaps A
    assert g(None, vp(1 << 22), vp(1 << 24), 16, 16, 16, None) == 1
    assert g(None, None, None, 0, 16, 16, None) == 0                          # empty: nothing to do
    # the failure-path self-check takes limits of 1 ns .. 1 s only
    cuda_lib.hstu_attn_selfcheck_wait_timeout.argtypes = [ctypes.c_uint64, vp]
    assert cuda_lib.hstu_attn_selfcheck_wait_timeout(0, None) == 1
    assert cuda_lib.hstu_attn_selfcheck_wait_timeout(2_000_000_000, None) == 1


def test_zero_rows_need_no_pointers(cuda_lib):
    """With no query rows nothing is read or written: NULL token pointers are accepted."""
    assert _fwd(cuda_lib, q=None, k=None, v=None, out=None, total=0, B=3) == 0
    assert _fwd(cuda_lib, q=None, k=None, v=None, out=None, off=None, total=0, B=0) == 0


def test_host_validation_bwd(cuda_lib):
    """The backward entry rejects bad sizes, misalignment and overlapping gradients on the host."""
    vp = ctypes.c_void_p
    f = cuda_lib.hstu_attn_bwd
    i32, f32 = ctypes.c_int32, ctypes.c_float
    f.argtypes = [vp] * 6 + [i32] * 5 + [f32, f32] + [vp] * 4
    mb = 1 << 20

    def call(q=mb, k=2 * mb, v=3 * mb, do=4 * mb, dq=5 * mb, dk=6 * mb, dv=7 * mb, d=64, N=1.0, B=1, total=16):
        return f(vp(q), vp(k), vp(v), vp(do), vp(4096), None, B, 2, d, total, 16, 1.0, N, vp(dq), vp(dk), vp(dv), None)

    assert call(d=48) == 2
    assert call(N=0.0) == 1
    assert call(B=-1) == 1
    assert call(do=None) == 1
    assert call(dk=None) == 1
    assert call(dv=4 * mb) == 1          # dv overlaps dout
    assert call(dk=5 * mb) == 1          # dk overlaps dq
    assert call(dq=mb + 64) == 1         # dq overlaps q
    assert call(do=4 * mb + 8) == 2      # misaligned dout
    assert call(q=None, k=None, v=None, do=None, dq=None, dk=None, dv=None, total=0) == 0
