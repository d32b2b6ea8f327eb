"""The allocation-free decode entry point, through the C ABI.

cr_w4a8_linear_decode_noalloc serves callers that cannot allocate device
memory during the call (a serving loop whose device memory all belongs to its
own allocator, a real-time path that cannot take an allocation's
synchronisation): it keeps the quantised activations in a scratch array the
library reserves statically on each device.  Its output must equal that of cr_w4a8_linear,
the entry point that takes caller-allocated scratch, on consecutive calls
that reuse (and so inherit the contents of) that static scratch.

This file is named so that pytest collects it last."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import w4a8_codebook_quantized_b200 as cr
from w4a8_codebook_quantized_b200 import inputs

from gpu_util import assert_output_close, bf16_dev, dev, host

pytestmark = pytest.mark.gpu


def _noalloc(L, x, layer_dev, M, N, K, out, kind, bias=None):
    q, s, cb, ws = layer_dev
    code = cr.CR_OUT_BF16 if kind == "bf16" else cr.CR_OUT_F32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.cr_w4a8_linear_decode_noalloc(x.data_ptr(), q.data_ptr(), s.data_ptr(), cb.data_ptr(), ws.data_ptr(),
                                           None if bias is None else bias.data_ptr(), M, N, K, 127, code,
                                           out.data_ptr(), stream)


def test_noalloc_decode_matches_linear_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = cr.lib()
    # consecutive calls with different shapes: the second one runs on scratch
    # that still holds the first call's activations
    for M, N, K, kind, seed in [(8, 4096, 4096, "bf16", 101), (3, 1000, 12288, "bf16", 102),
                                (1, 256, 256, "f32", 103), (5, 2048, 8192, "bf16", 104)]:
        layer = inputs.layer(N, K, seed)
        layer_dev = (dev(layer.qdata), dev(layer.srel), dev(layer.codebook), dev(layer.s_channel))
        x = bf16_dev(inputs.activations(M, K, seed))
        dt = torch.bfloat16 if kind == "bf16" else torch.float32
        out = torch.empty(M, N, dtype=dt, device="cuda")
        assert _noalloc(L, x, layer_dev, M, N, K, out, kind) == cr.CR_OK
        ref = cr.cr_w4a8_linear(x, *layer_dev, out_dtype=dt)
        torch.cuda.synchronize()
        assert_output_close(host(out), host(ref), kind)


def test_noalloc_decode_matches_the_oracle_with_bias_and_at_the_scratch_limit():
    """Against the CPU oracle, bit for bit, with a bias, and at the largest
    size the static scratch holds (M = 8, K = CR_MAX_K), twice in a row."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = cr.lib()
    for M, N, K, kind, seed in [(6, 300, 2048, "f32", 111), (8, 48, 131072, "bf16", 112),
                                (8, 48, 131072, "bf16", 113)]:
        layer = inputs.layer(N, K, seed, with_bias=True)
        layer_dev = (dev(layer.qdata), dev(layer.srel), dev(layer.codebook), dev(layer.s_channel))
        x_np = inputs.activations(M, K, seed)
        dt = torch.bfloat16 if kind == "bf16" else torch.float32
        out = torch.empty(M, N, dtype=dt, device="cuda")
        assert _noalloc(L, bf16_dev(x_np), layer_dev, M, N, K, out, kind, dev(layer.bias)) == cr.CR_OK
        torch.cuda.synchronize()
        ref = oracle.linear(x_np, layer.qdata, layer.srel, layer.codebook, layer.s_channel, layer.bias,
                            out=kind, threads=8)
        assert_output_close(host(out), ref["y"], kind)


def test_noalloc_rejects_prefill_sizes():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = cr.lib()
    a = torch.empty(64, dtype=torch.uint8, device="cuda")
    p = a.data_ptr()
    # M beyond the decode range: the padded activations would not fit the scratch
    assert L.cr_w4a8_linear_decode_noalloc(p, p, p, p, p, None, 9, 16, 256, 127, 0, p, None) == cr.CR_ERR_UNSUPPORTED
    assert L.cr_w4a8_linear_decode_noalloc(p, p, p, p, p, None, 2, 16, 131072 + 256, 127, 0, p,
                                           None) == cr.CR_ERR_UNSUPPORTED
    assert L.cr_w4a8_linear_decode_noalloc(p, p, p, p, p, None, 0, 16, 256, 127, 0, p, None) == cr.CR_OK
    # N beyond the int range of the kernel's row count
    assert L.cr_w4a8_linear_decode_noalloc(p, p, p, p, p, None, 2, 2 ** 31, 256, 127, 0, p,
                                           None) == cr.CR_ERR_UNSUPPORTED
