"""GPU parity at the benchmark's full sizes, in the launch configuration the
benchmark times (cr_w4a8_linear: rotate+quant, then the GEMV for M <= 8 or
the decode transient + tcgen05 GEMM for M > 8).

The int8 activations and scales and the int8 weight grid are compared in
full; the int32 accumulators and outputs are compared in full where the
oracle finishes in seconds (decode batches) and on a seeded sample of token
rows (first and last row included) otherwise -- every row of the output is
independent of the others, so a row sample checks whole rows exactly."""
import os

import numpy as np
import pytest
import torch

import oracle
import w4a8_codebook_quantized_b200 as cr
from w4a8_codebook_quantized_b200 import inputs

from gpu_util import assert_output_close, bf16_dev, dev, host

pytestmark = pytest.mark.gpu
THREADS = max(1, min(32, os.cpu_count() or 1))
SAMPLE_ROWS = 48


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cr.lib()
    yield
    cr.cr_check_device_error()


def _run_case(name):
    case = inputs.CASES[name]
    M, N, K = case.M, case.N, case.K
    layer = inputs.layer(N, K, case.seed)
    x = inputs.activations(M, K, case.seed, case.dist)
    q, s, cb, ws = dev(layer.qdata), dev(layer.srel), dev(layer.codebook), dev(layer.s_channel)
    xd = bf16_dev(x)
    rows = cr.gemv_rows(M) if M <= 8 else M
    xq = torch.empty(rows, K, dtype=torch.int8, device="cuda")
    xs = torch.empty(rows, dtype=torch.float32, device="cuda")
    y = cr.cr_w4a8_linear(xd, q, s, cb, ws, xq_work=xq, xs_work=xs)
    fn = cr.cr_w4a8_gemv if M <= 8 else cr.cr_w4a8_gemm
    _, acc = fn(xq, xs, q, s, cb, ws, m=M, acc_out=True)
    torch.cuda.synchronize()

    # activations in full
    xq_r, xs_r = oracle.rotate_quant_act(x, rows, 127)
    assert np.array_equal(host(xs).view(np.uint32), xs_r.view(np.uint32))
    assert np.array_equal(host(xq), xq_r)
    # weight grid in full
    w8_r = oracle.decode_w8(layer.qdata, layer.srel, layer.codebook)
    assert np.array_equal(host(cr.cr_w4a8_decode_int8(q, s, cb)), w8_r)
    # accumulators and outputs: all rows, or a sample of whole rows
    if M <= 64:
        sel = np.arange(M)
    else:
        rng = np.random.default_rng(case.seed)
        sel = np.unique(np.concatenate([[0, M - 1], rng.choice(M, SAMPLE_ROWS, replace=False)]))
    acc_r = oracle.gemm_s32(xq_r[sel], w8_r, THREADS)
    y_r = oracle.epilogue(acc_r, xs_r[sel], layer.s_channel, None, "bf16")
    idx = torch.from_numpy(sel).cuda()
    assert np.array_equal(host(acc.index_select(0, idx)), acc_r)
    assert_output_close(host(y.index_select(0, idx)), y_r, "bf16")


@pytest.mark.parametrize("name", ["c1_decode_m1_1k", "c2_decode_m8_4k", "c5_m1_8k", "c5_m2_8k", "c5_m4_8k",
                                  "c5_m8_8k"])
def test_decode_configs_full(name):
    _run_case(name)


@pytest.mark.parametrize("name", ["c3_prefill_2k_4k", "c4_mlp_up", "c4_mlp_down", "c5_m16384_8k"])
def test_prefill_configs_sampled(name):
    _run_case(name)


def test_c2_gemv_equals_gemm_bitwise():
    case = inputs.CASES["c2_decode_m8_4k"]
    layer = inputs.layer(case.N, case.K, case.seed)
    x = bf16_dev(inputs.activations(case.M, case.K, case.seed))
    q, s, cb, ws = dev(layer.qdata), dev(layer.srel), dev(layer.codebook), dev(layer.s_channel)
    xq, xs = cr.cr_rotate_quant_act(x, 8, 127)
    o1, a1 = cr.cr_w4a8_gemv(xq, xs, q, s, cb, ws, acc_out=True)
    o2, a2 = cr.cr_w4a8_gemm(xq, xs, q, s, cb, ws, acc_out=True)
    assert torch.equal(a1, a2)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
