"""The C ABI without a GPU: the library loads, exports every entry point the
header declares, and rejects bad arguments before touching any device."""
import ctypes
import os
import re

import pytest

import w4a8_codebook_quantized_b200 as cr
from w4a8_codebook_quantized_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cr_w4a8.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return cr.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(cr_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("cr_rotate_quant_act", "cr_w4a8_decode_int8", "cr_w4a8_gemm", "cr_w4a8_gemv", "cr_epilogue",
              "cr_w4a8_linear", "cr_status_string", "cr_check_device_error", "cr_version",
              "cr_w4a8_gemv_grouped", "cr_w4a8_linear_grouped", "cr_w4a8_gemm_swiglu", "cr_w4a8_gemv_swiglu",
              "cr_w4a8_linear_swiglu", "cr_interleave_rows", "cr_w4a8_quantize_rotated", "cr_w4a8_assign_codes",
              "cr_w4a8_ste_backward", "cr_w4a8_dequant_t_bf16", "cr_w4a8_plan_create", "cr_w4a8_plan_forward",
              "cr_w4a8_plan_forward_host", "cr_w4a8_plan_destroy", "cr_selftest_wait_timeout", "cr_gemm_s8",
              "cr_w4a8_plan_bind_host", "cr_w4a8_host_call_run", "cr_w4a8_host_call_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), name
    out = os.popen(f"nm -D --defined-only {cr.library_path()}").read()
    exported = set(re.findall(r" T (cr_\w+)", out))
    assert set(_declared()) <= exported
    # nothing else leaks out under the cr_ prefix
    assert exported == set(_declared())


def test_library_is_built_for_sm100a_only():
    out = os.popen(f"cuobjdump --list-elf {cr.library_path()} 2>&1").read()
    assert "sm_100a" in out
    assert not re.search(r"sm_(?!100a)\d+", out)


def test_status_strings(L):
    for s in range(7):
        assert cr.cr_status_string(s)
    assert cr.cr_status_string(99) == "unknown status"
    assert cr.cr_version().count(".") == 2


P = ctypes.c_void_p
A16 = 0x10000  # a 16-byte aligned stand-in address; never dereferenced on these paths
MIS = 0x10008  # 8-byte aligned only


def test_rotate_quant_validation(L):
    f = L.cr_rotate_quant_act
    assert f(A16, -1, 256, 1, 127, A16, A16, None) == cr.CR_ERR_INVALID_ARG
    assert f(A16, 2, 256, 1, 127, A16, A16, None) == cr.CR_ERR_INVALID_ARG      # MP < M
    assert f(A16, 1, 256, 1, 0, A16, A16, None) == cr.CR_ERR_INVALID_ARG        # qmax
    assert f(A16, 1, 256, 1, 128, A16, A16, None) == cr.CR_ERR_INVALID_ARG
    assert f(A16, 1, 128, 1, 127, A16, A16, None) == cr.CR_ERR_UNSUPPORTED      # K % 256
    assert f(A16, 1, 0, 1, 127, A16, A16, None) == cr.CR_ERR_UNSUPPORTED
    assert f(A16, 1, 131072 + 256, 1, 127, A16, A16, None) == cr.CR_ERR_UNSUPPORTED
    assert f(None, 1, 256, 1, 127, A16, A16, None) == cr.CR_ERR_INVALID_ARG
    assert f(MIS, 1, 256, 1, 127, A16, A16, None) == cr.CR_ERR_ALIGNMENT
    assert f(A16, 1, 256, 1, 127, MIS, A16, None) == cr.CR_ERR_ALIGNMENT
    assert f(None, 0, 256, 0, 127, None, None, None) == cr.CR_OK                # empty


def test_decode_validation(L):
    f = L.cr_w4a8_decode_int8
    assert f(A16, A16, A16, -1, 256, A16, None) == cr.CR_ERR_INVALID_ARG
    assert f(A16, A16, A16, 4, 272, A16, None) == cr.CR_ERR_UNSUPPORTED
    assert f(None, A16, A16, 4, 256, A16, None) == cr.CR_ERR_INVALID_ARG
    assert f(A16, MIS, A16, 4, 256, A16, None) == cr.CR_ERR_ALIGNMENT
    assert f(None, None, None, 0, 256, None, None) == cr.CR_OK


def test_bound_host_call_validation(L):
    call = ctypes.c_void_p(1)
    assert L.cr_w4a8_plan_bind_host(None, A16, 2, A16, A16, A16, A16, A16, ctypes.byref(call)) == cr.CR_ERR_INVALID_ARG
    assert call.value is None  # written NULL on error
    assert L.cr_w4a8_plan_bind_host(None, A16, 2, A16, A16, A16, A16, A16, None) == cr.CR_ERR_INVALID_ARG
    assert L.cr_w4a8_host_call_run(None, None) == cr.CR_ERR_INVALID_ARG
    assert L.cr_w4a8_host_call_destroy(None) == cr.CR_OK


def test_gemm_s8_validation(L):
    f = L.cr_gemm_s8
    assert f(A16, A16, A16, A16, None, -1, 8, 256, 0, A16, None, None) == cr.CR_ERR_INVALID_ARG
    assert f(A16, A16, A16, A16, None, 4, 8, 320, 0, A16, None, None) == cr.CR_ERR_UNSUPPORTED
    assert f(A16, A16, None, A16, None, 4, 8, 256, 0, A16, None, None) == cr.CR_ERR_INVALID_ARG
    assert f(A16, A16, MIS, A16, None, 4, 8, 256, 0, A16, None, None) == cr.CR_ERR_ALIGNMENT
    assert f(A16, A16, A16, A16, None, 4, 8, 256, 3, A16, None, None) == cr.CR_ERR_INVALID_ARG
    assert f(None, None, None, None, None, 0, 8, 256, 0, None, None, None) == cr.CR_OK


@pytest.mark.parametrize("name", ["cr_w4a8_gemm", "cr_w4a8_gemv"])
def test_contraction_validation(L, name):
    f = getattr(L, name)
    ok = [A16] * 7

    def call(M=4, N=8, K=256, dtype=0, ptrs=None, out=A16, acc=None):
        p = ptrs or ok
        return f(*p, M, N, K, dtype, out, acc, None)

    assert call(M=-1) == cr.CR_ERR_INVALID_ARG
    assert call(dtype=7) == cr.CR_ERR_INVALID_ARG
    assert call(K=320) == cr.CR_ERR_UNSUPPORTED
    assert call(out=None) == cr.CR_ERR_INVALID_ARG
    bad = list(ok)
    bad[3] = MIS
    assert call(ptrs=bad) == cr.CR_ERR_ALIGNMENT
    nob = list(ok)
    nob[6] = None  # bias is optional: fine
    assert call(ptrs=nob, M=0) == cr.CR_OK
    assert call(acc=MIS) == cr.CR_ERR_ALIGNMENT
    assert call(M=0) == cr.CR_OK and call(N=0) == cr.CR_OK
    if name == "cr_w4a8_gemv":
        assert call(M=9) == cr.CR_ERR_UNSUPPORTED


def test_epilogue_and_linear_validation(L):
    assert L.cr_epilogue(A16, A16, A16, None, -1, 4, 0, A16, None) == cr.CR_ERR_INVALID_ARG
    assert L.cr_epilogue(A16, A16, A16, None, 2, 4, 3, A16, None) == cr.CR_ERR_INVALID_ARG
    assert L.cr_epilogue(A16, MIS, A16, None, 2, 4, 0, A16, None) == cr.CR_ERR_ALIGNMENT
    assert L.cr_epilogue(None, None, None, None, 0, 4, 0, None, None) == cr.CR_OK
    f = L.cr_w4a8_linear
    assert f(A16, A16, A16, A16, A16, None, 2, 8, 256, 0, 0, A16, A16, A16, None) == cr.CR_ERR_INVALID_ARG
    assert f(A16, A16, A16, A16, A16, None, 2, 8, 384, 127, 0, A16, A16, A16, None) == cr.CR_ERR_UNSUPPORTED
    assert f(None, A16, A16, A16, A16, None, 2, 8, 256, 127, 0, A16, A16, A16, None) == cr.CR_ERR_INVALID_ARG
    assert f(MIS, A16, A16, A16, A16, None, 2, 8, 256, 127, 0, A16, A16, A16, None) == cr.CR_ERR_ALIGNMENT


def _layers(*specs):
    """A cr_w4a8_layer array; each spec is a dict of field overrides."""
    arr = (cr.CrLayer * max(1, len(specs)))()
    for i, sp in enumerate(specs):
        f = dict(qdata=A16, srel=A16, s_channel=A16, bias=None, N=8, out=A16, acc_out=None)
        f.update(sp)
        arr[i] = cr.CrLayer(**f)
    return arr


def test_grouped_validation(L):
    g = L.cr_w4a8_gemv_grouped
    two = _layers({}, {"N": 16})
    assert g(A16, A16, A16, 4, 256, two, 0, 0, None) == cr.CR_ERR_INVALID_ARG            # no layers
    assert g(A16, A16, A16, 4, 256, _layers(*[{}] * 5), 5, 0, None) == cr.CR_ERR_INVALID_ARG  # > CR_MAX_LAYERS
    assert g(A16, A16, A16, 4, 256, None, 1, 0, None) == cr.CR_ERR_INVALID_ARG
    assert g(A16, A16, A16, 9, 256, two, 2, 0, None) == cr.CR_ERR_UNSUPPORTED             # M > 8
    assert g(A16, A16, A16, 4, 320, two, 2, 0, None) == cr.CR_ERR_UNSUPPORTED             # K % 256
    assert g(A16, A16, A16, 4, 256, two, 2, 5, None) == cr.CR_ERR_INVALID_ARG             # out dtype
    assert g(A16, A16, A16, 4, 256, _layers({}, {"srel": MIS}), 2, 0, None) == cr.CR_ERR_ALIGNMENT
    assert g(A16, A16, A16, 4, 256, _layers({}, {"out": None}), 2, 0, None) == cr.CR_ERR_INVALID_ARG
    assert g(A16, A16, A16, 4, 256, _layers({"N": -1}), 1, 0, None) == cr.CR_ERR_INVALID_ARG
    assert g(A16, A16, MIS, 4, 256, two, 2, 0, None) == cr.CR_ERR_ALIGNMENT               # codebook
    # empty layers may carry null pointers; an all-empty call or M == 0 does nothing
    empty = _layers({"N": 0, "qdata": None, "srel": None, "s_channel": None, "out": None})
    assert g(A16, A16, A16, 4, 256, empty, 1, 0, None) == cr.CR_OK
    assert g(None, None, None, 0, 256, two, 2, 0, None) == cr.CR_OK
    f = L.cr_w4a8_linear_grouped
    assert f(A16, A16, 2, 256, two, 2, 0, 0, A16, A16, None) == cr.CR_ERR_INVALID_ARG       # act_qmax
    assert f(A16, A16, 2, 256, _layers({"acc_out": A16}), 1, 127, 0, A16, A16, None) == cr.CR_ERR_INVALID_ARG
    assert f(None, A16, 2, 256, two, 2, 127, 0, A16, A16, None) == cr.CR_ERR_INVALID_ARG
    assert f(MIS, A16, 2, 256, two, 2, 127, 0, A16, A16, None) == cr.CR_ERR_ALIGNMENT
    assert f(A16, A16, 2, 256, two, 2, 127, 0, MIS, A16, None) == cr.CR_ERR_ALIGNMENT
    assert f(None, A16, 2, 256, empty, 1, 127, 0, None, None, None) == cr.CR_OK


@pytest.mark.parametrize("name", ["cr_w4a8_gemm_swiglu", "cr_w4a8_gemv_swiglu"])
def test_swiglu_contraction_validation(L, name):
    f = getattr(L, name)
    ok = [A16] * 7

    def call(M=4, N=8, K=256, dtype=0, ptrs=None, out=A16):
        return f(*(ptrs or ok), M, N, K, dtype, out, None)

    assert call(N=7) == cr.CR_ERR_INVALID_ARG         # gate/up pairs need an even N
    assert call(M=-1) == cr.CR_ERR_INVALID_ARG
    assert call(dtype=2) == cr.CR_ERR_INVALID_ARG
    assert call(K=320) == cr.CR_ERR_UNSUPPORTED
    assert call(out=None) == cr.CR_ERR_INVALID_ARG
    assert call(out=MIS) == cr.CR_ERR_ALIGNMENT
    assert call(M=0) == cr.CR_OK and call(N=0) == cr.CR_OK
    if name == "cr_w4a8_gemv_swiglu":
        assert call(M=9) == cr.CR_ERR_UNSUPPORTED
    g = L.cr_w4a8_linear_swiglu
    assert g(A16, A16, A16, A16, A16, None, 2, 7, 256, 127, 0, A16, A16, A16, None) == cr.CR_ERR_INVALID_ARG
    assert g(A16, A16, A16, A16, A16, None, 2, 8, 256, 0, 0, A16, A16, A16, None) == cr.CR_ERR_INVALID_ARG
    assert g(MIS, A16, A16, A16, A16, None, 2, 8, 256, 127, 0, A16, A16, A16, None) == cr.CR_ERR_ALIGNMENT
    assert g(None, None, None, None, None, None, 0, 8, 256, 127, 0, None, None, None, None) == cr.CR_OK


def test_interleave_rows_validation(L):
    f = L.cr_interleave_rows
    assert f(A16, 0x20000, 3, 16, None) == cr.CR_ERR_INVALID_ARG      # odd row count
    assert f(A16, 0x20000, -2, 16, None) == cr.CR_ERR_INVALID_ARG
    assert f(A16, 0x20000, 2, -1, None) == cr.CR_ERR_INVALID_ARG
    assert f(None, 0x20000, 2, 16, None) == cr.CR_ERR_INVALID_ARG
    assert f(A16, A16 + 16, 2, 16, None) == cr.CR_ERR_INVALID_ARG     # overlapping buffers
    assert f(None, None, 0, 16, None) == cr.CR_OK and f(None, None, 2, 0, None) == cr.CR_OK
    assert f(A16, 0x20000, 2 ** 40, 2 ** 40, None) == cr.CR_ERR_INVALID_ARG  # size overflows


def test_quantiser_validation(L):
    f, g = L.cr_w4a8_quantize_rotated, L.cr_w4a8_assign_codes
    assert f(A16, A16, -1, 16, A16, A16, A16, None) == cr.CR_ERR_INVALID_ARG
    assert f(A16, A16, 4, 24, A16, A16, A16, None) == cr.CR_ERR_UNSUPPORTED      # K % 16
    assert f(A16, A16, 4, 0, A16, A16, A16, None) == cr.CR_ERR_UNSUPPORTED
    assert f(A16, A16, 4, 131072 + 16, A16, A16, A16, None) == cr.CR_ERR_UNSUPPORTED
    assert f(None, A16, 4, 16, A16, A16, A16, None) == cr.CR_ERR_INVALID_ARG
    assert f(A16, A16, 4, 16, A16, MIS, A16, None) == cr.CR_ERR_ALIGNMENT
    assert f(None, None, 0, 16, None, None, None, None) == cr.CR_OK
    assert g(A16, A16, A16, A16, None, 4, 24, A16, None) == cr.CR_ERR_UNSUPPORTED
    assert g(A16, A16, A16, A16, MIS, 4, 16, A16, None) == cr.CR_ERR_ALIGNMENT   # rand
    assert g(A16, None, A16, A16, None, 4, 16, A16, None) == cr.CR_ERR_INVALID_ARG
    assert g(None, None, None, None, None, 0, 16, None, None) == cr.CR_OK


def test_backward_validation(L):
    f, g = L.cr_w4a8_ste_backward, L.cr_w4a8_dequant_t_bf16
    assert f(A16, A16, A16, A16, A16, -1, 8, 256, A16, None) == cr.CR_ERR_INVALID_ARG
    assert f(A16, A16, A16, A16, A16, 4, 12, 256, A16, None) == cr.CR_ERR_UNSUPPORTED   # N % 8
    assert f(A16, A16, A16, A16, A16, 4, 8, 320, A16, None) == cr.CR_ERR_UNSUPPORTED    # K % 256
    assert f(None, A16, A16, A16, A16, 4, 8, 256, A16, None) == cr.CR_ERR_INVALID_ARG
    assert f(A16, A16, A16, A16, A16, 4, 8, 256, MIS, None) == cr.CR_ERR_ALIGNMENT
    assert f(None, None, None, None, None, 0, 8, 256, None, None) == cr.CR_OK
    assert g(A16, A16, A16, A16, 12, 256, A16, None) == cr.CR_ERR_UNSUPPORTED
    assert g(A16, A16, MIS, A16, 8, 256, A16, None) == cr.CR_ERR_ALIGNMENT
    assert g(None, None, None, None, 0, 256, None, None) == cr.CR_OK


def test_plan_validation(L):
    plan = ctypes.c_void_p()
    f = L.cr_w4a8_plan_create
    assert f(A16, A16, A16, A16, None, 8, 256, 0, 0, ctypes.byref(plan)) == cr.CR_ERR_INVALID_ARG   # act_qmax
    assert f(A16, A16, A16, A16, None, 8, 256, 127, 9, ctypes.byref(plan)) == cr.CR_ERR_INVALID_ARG  # out dtype
    assert f(A16, A16, A16, A16, None, 8, 320, 127, 0, ctypes.byref(plan)) == cr.CR_ERR_UNSUPPORTED
    assert f(None, A16, A16, A16, None, 8, 256, 127, 0, ctypes.byref(plan)) == cr.CR_ERR_INVALID_ARG
    assert f(A16, MIS, A16, A16, None, 8, 256, 127, 0, ctypes.byref(plan)) == cr.CR_ERR_ALIGNMENT
    assert f(A16, A16, A16, A16, None, 8, 256, 127, 0, None) == cr.CR_ERR_INVALID_ARG
    assert L.cr_w4a8_plan_forward(None, A16, 2, A16, A16, A16, None) == cr.CR_ERR_INVALID_ARG
    assert L.cr_w4a8_plan_forward_host(None, A16, 2, A16, A16, A16, A16, A16, None) == cr.CR_ERR_INVALID_ARG
    assert L.cr_w4a8_plan_destroy(None) == cr.CR_OK


def test_int8_peak_validation(L):
    ops = ctypes.c_double(-1.0)
    assert L.cr_mma_i8_peak(0, ctypes.byref(ops), None) == cr.CR_ERR_INVALID_ARG
    assert L.cr_mma_i8_peak((1 << 20) + 1, ctypes.byref(ops), None) == cr.CR_ERR_INVALID_ARG
    assert L.cr_mma_i8_peak(16, None, None) == cr.CR_ERR_INVALID_ARG
    assert ops.value == -1.0


def test_selftest_validation(L):
    assert L.cr_selftest_wait_timeout(10, None) == cr.CR_ERR_INVALID_ARG        # below 1 ms
    assert L.cr_selftest_wait_timeout(2 * 10 ** 9, None) == cr.CR_ERR_INVALID_ARG  # above 1 s


def test_valid_call_without_a_gpu_fails_loudly(L):
    """On a machine with no usable sm_100 device a well-formed call reports
    CR_ERR_NO_DEVICE instead of computing anything anywhere else."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert L.cr_w4a8_decode_int8(A16, A16, A16, 4, 256, A16, None) == cr.CR_ERR_NO_DEVICE
    assert L.cr_check_device_error(None) == cr.CR_ERR_NO_DEVICE
    with pytest.raises(ValueError):
        cr.cr_w4a8_decode_int8(torch.zeros(4, 128, dtype=torch.uint8), torch.zeros(4, 16, dtype=torch.uint8),
                               torch.zeros(16))
