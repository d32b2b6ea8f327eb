"""GPU parity at edge cases: exact rounding ties through the rotation, SwiGLU
gates so negative that exp(-g) overflows fp32, the library's device memory
around prefill calls and the caller-workspace variants, and calls on a
device other than the current one."""
import math

import numpy as np
import pytest
import torch

import oracle
import w4a8_codebook_quantized_b200 as cr
from w4a8_codebook_quantized_b200 import inputs

from gpu_util import assert_output_close, assert_swiglu_close, bf16_dev, dev, host

pytestmark = pytest.mark.gpu

H4 = np.array([[1, 1, 1, -1], [1, 1, -1, 1], [1, -1, 1, 1], [-1, 1, 1, 1]], dtype=np.float64)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cr.lib()
    yield
    cr.cr_check_device_error()


def _h256():
    h = np.ones((1, 1))
    while h.shape[0] < 256:
        h = np.kron(h, H4)
    return h / 16.0


def _x_for_rotated(r):
    """bf16 bits of x with x . H = r block-wise (H is symmetric and H . H = I,
    so x = r . H); asserts that x is exactly representable in bf16, so that
    the rotation of x gives r back exactly (every butterfly partial sum of
    these small multiples of 1/32 is exact in fp32)."""
    M, K = r.shape
    H = _h256()
    x = np.concatenate([r[:, b:b + 256] @ H for b in range(0, K, 256)], axis=1)
    bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    back = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(back, x), "the test's x is not exact in bf16"
    return bits


@pytest.mark.parametrize("reps", [1, 10])
@pytest.mark.parametrize("qmax", [64, 127])
def test_rotate_quant_exact_ties(qmax, reps):
    """Rotated rows with amax == qmax (scale exactly 1) and half-integer
    entries: every entry is an exact tie of rint, which goes to the even
    integer (ai-toolkit convrot_w4a8_quant.py, w4a8_act_quant_kernel,
    libdevice rint).  The device's division-free rounding must take its exact
    path here and agree with the oracle bit for bit: as a short batch (4 rows)
    and, with the rows repeated, as a 40-row batch (the packed form, where a
    block pair's two halves carry the ties of blocks 0 and 1)."""
    K = 512
    r = np.zeros((4, K), np.float64)
    if qmax == 64:
        # row 0: the max and ties in block 0, more ties in block 1
        r[0, [0, 5, 17, 100, 200, 255]] = [64, 2.5, -3.5, 0.5, 1.5, -0.5]
        r[0, 256 + 3], r[0, 256 + 40] = 5.5, -62.5
        # row 1: the max is negative; ties up to 63.5 (rounds to 64)
        r[1, [7, 9, 11]] = [-64, 4.5, 6.5]
        r[1, 256 + np.array([20, 21, 30, 31])] = [63.5, -7.5, 0.5, -1.5]
        expect = {(0, 0): 64, (0, 5): 2, (0, 17): -4, (0, 100): 0, (0, 200): 2, (0, 255): 0,
                  (0, 259): 6, (0, 296): -62, (1, 7): -64, (1, 9): 4, (1, 11): 6, (1, 276): 64, (1, 277): -8,
                  (1, 286): 0, (1, 287): -2}
    else:
        # the max alone in block 0, the ties in block 1 (keeps x exact in bf16)
        r[0, 0] = 127
        r[0, 256 + np.array([1, 2, 3, 4])] = [2.5, -3.5, 0.5, 1.5]
        r[1, 255] = -127
        r[1, 256 + np.array([8, 9, 10, 11])] = [-0.5, -2.5, 4.5, 0.5]
        expect = {(0, 0): 127, (0, 257): 2, (0, 258): -4, (0, 259): 0, (0, 260): 2,
                  (1, 255): -127, (1, 264): 0, (1, 265): -2, (1, 266): 4, (1, 267): 0}
    # row 2: all zero (scale 1); row 3: row 0 doubled, so its scale is 2 and
    # r / scale gives row 0's ties again
    r[3] = 2 * r[0]
    r = np.tile(r, (reps, 1))
    x = _x_for_rotated(r)
    xq_r, xs_r = oracle.rotate_quant_act(x, 4 * reps, qmax)
    for rep in range(reps):
        for (m, k), q in expect.items():
            assert int(xq_r[4 * rep + m, k]) == q, (rep, m, k, int(xq_r[4 * rep + m, k]), q)
    assert xs_r[0] == 1.0 and xs_r[1] == 1.0 and xs_r[2] == 1.0
    xq, xs = cr.cr_rotate_quant_act(bf16_dev(x), 4 * reps, qmax)
    torch.cuda.synchronize()
    assert np.array_equal(host(xs).view(np.uint32), xs_r.view(np.uint32))
    assert np.array_equal(host(xq), xq_r)


@pytest.mark.parametrize("M,K", [(8, 4096), (64, 4096), (20, 768), (4, 16384), (40, 12288)])
def test_rotate_quant_wide_exponents(M, K):
    """bf16 rows whose values spread over 2^-24 .. 2^24, so that the fp32
    partial sums of the butterfly round (on the configs' activations they are
    mostly exact): the row scales (the rounded maximum of each rotated row
    over qmax) and every quantised byte must equal the oracle's, in both
    kernel forms (short batches and the packed pairs)."""
    rng = np.random.default_rng(M * 7 + K)
    vals = rng.choice([-1.0, 1.0], size=(M, K)) * np.exp2(rng.integers(-24, 25, size=(M, K))) * \
        rng.uniform(1.0, 2.0, size=(M, K))
    x = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    mp = cr.gemv_rows(M) if M <= 8 else M
    xq, xs = cr.cr_rotate_quant_act(bf16_dev(x), mp, 127)
    torch.cuda.synchronize()
    xq_r, xs_r = oracle.rotate_quant_act(x, mp, 127)
    assert np.array_equal(host(xs).view(np.uint32), xs_r.view(np.uint32))
    assert np.array_equal(host(xq), xq_r)


def _very_negative_gate_layer(F, K, seed):
    """An interleaved gate/up layer whose epilogue values are dominated by
    the bias: gates g in about [-90.5, -85] (e^-g overflows fp32 below -88.7,
    and 1 + e^-g exceeds 2^126 above it, while silu(g) * u = g e^g u / (1 + e^g)
    stays a normal fp32 number) and up values u in about [0.5, 2]."""
    ly = inputs.layer(2 * F, K, seed)
    rng = np.random.default_rng(seed)
    s_channel = np.full(2 * F, 1e-9, np.float32)
    bias = np.empty(2 * F, np.float32)
    bias[0::2] = rng.uniform(-90.5, -85.0, F)
    bias[1::2] = rng.uniform(0.5, 2.0, F)
    return ly.qdata, ly.srel, ly.codebook, s_channel, bias


@pytest.mark.parametrize("fn,M,F,K", [("gemv", 5, 512, 1024), ("gemm", 300, 256, 512)])
@pytest.mark.parametrize("kind", ["bf16", "f32"])
def test_swiglu_very_negative_gates(fn, M, F, K, kind):
    """silu(g) * u for gates where e^-g overflows or where 1 + e^-g lies
    beyond 2^126: the device result must be the small normal number the
    oracle computes (in double), within one unit in the last place, with no
    absolute floor below which errors would pass."""
    qd, sr, cb, ws, bias = _very_negative_gate_layer(F, K, M + F + K)
    x = inputs.activations(M, K, M + K)
    xq_r, xs_r = oracle.rotate_quant_act(x, None, 127)
    acc_r = oracle.gemm_s32(xq_r, oracle.decode_w8(qd, sr, cb))
    y_r = oracle.epilogue_swiglu(acc_r, xs_r, ws, bias, kind)
    ref = y_r.astype(np.float64) if kind == "f32" else \
        ((y_r.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    assert np.all(np.abs(ref) > 2.0 ** -126), "the case should stay in the normal range"
    dt = torch.bfloat16 if kind == "bf16" else torch.float32
    call = cr.cr_w4a8_gemv_swiglu if fn == "gemv" else cr.cr_w4a8_gemm_swiglu
    out = call(dev(xq_r), dev(xs_r), dev(qd), dev(sr), dev(cb), dev(ws), dev(bias), out_dtype=dt)
    torch.cuda.synchronize()
    got = host(out)
    assert_swiglu_close(got, y_r, kind)
    g = got.astype(np.float64) if kind == "f32" else ((got.astype(np.uint32) << 16).view(np.float32)
                                                      .astype(np.float64))
    rel = 2.0 ** -7 if kind == "bf16" else 4e-6
    assert np.all(np.abs(g - ref) <= rel * np.abs(ref)), np.max(np.abs(g - ref) / np.abs(ref))


# ---------------------------------------------------------------- device memory of the library

def _free_bytes():
    torch.cuda.synchronize()
    torch.cuda.synchronize()
    return torch.cuda.mem_get_info()[0]


def test_prefill_transient_goes_back_after_a_sync():
    """cr_w4a8_gemm takes its N*K weight transient from the library's pool
    and frees it at the end of the call; after a synchronisation the pool
    holds nothing, so the device's free memory is back where it was."""
    M, N, K = 512, 8192, 8192  # a 64 MiB transient
    layer = inputs.layer(N, K, 31)
    q, s, cb, ws = dev(layer.qdata), dev(layer.srel), dev(layer.codebook), dev(layer.s_channel)
    xq, xs = cr.cr_rotate_quant_act(bf16_dev(inputs.activations(M, K, 31)))
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    x = bf16_dev(inputs.activations(M, K, 32))
    xq_w = torch.empty(M, K, dtype=torch.int8, device="cuda")
    xs_w = torch.empty(M, dtype=torch.float32, device="cuda")
    for _ in range(2):  # a first call creates the side stream and the pool itself
        cr.cr_w4a8_gemm(xq, xs, q, s, cb, ws, out=out)
        cr.cr_w4a8_linear(x, q, s, cb, ws, out=out, xq_work=xq_w, xs_work=xs_w)
    free0 = _free_bytes()
    for _ in range(3):
        cr.cr_w4a8_gemm(xq, xs, q, s, cb, ws, out=out)
        cr.cr_w4a8_linear(x, q, s, cb, ws, out=out, xq_work=xq_w, xs_work=xs_w)
    free1 = _free_bytes()
    assert free0 - free1 < 4 * 2 ** 20, (free0 - free1) / 2 ** 20


@pytest.mark.parametrize("M,N,K", [(300, 1000, 768), (2048, 4096, 512), (5, 776, 2048)])
def test_workspace_variants_equal_and_allocate_nothing(M, N, K):
    """cr_w4a8_gemm_ws / cr_w4a8_linear_ws decode into the caller's w8_work:
    bit for bit the results of the pool-transient calls, the decoded grid of
    cr_w4a8_decode_int8 left in w8_work, and no change in free device memory
    even before any synchronisation."""
    layer = inputs.layer(N, K, M + N + K, with_bias=True)
    q, s, cb, ws, b = (dev(layer.qdata), dev(layer.srel), dev(layer.codebook), dev(layer.s_channel),
                       dev(layer.bias))
    x = bf16_dev(inputs.activations(M, K, M + K))
    rows = cr.gemv_rows(M) if M <= 8 else M
    xq_w = torch.empty(rows, K, dtype=torch.int8, device="cuda")
    xs_w = torch.empty(rows, dtype=torch.float32, device="cuda")
    w8 = torch.zeros(N, K, dtype=torch.int8, device="cuda")
    y_ref = cr.cr_w4a8_linear(x, q, s, cb, ws, b, xq_work=xq_w.clone(), xs_work=xs_w.clone())
    y = torch.empty_like(y_ref)
    free0 = _free_bytes()
    cr.cr_w4a8_linear_ws(x, q, s, cb, ws, w8, b, out=y, xq_work=xq_w, xs_work=xs_w)
    free1 = torch.cuda.mem_get_info()[0]  # no synchronisation in between
    torch.cuda.synchronize()
    assert free0 - free1 < 2 ** 20
    assert torch.equal(y, y_ref)
    if M > 8:
        assert torch.equal(w8, cr.cr_w4a8_decode_int8(q, s, cb))
        xq, xs = cr.cr_rotate_quant_act(x)
        o1, a1 = cr.cr_w4a8_gemm(xq, xs, q, s, cb, ws, b, acc_out=True)
        w8.zero_()
        o2, a2 = cr.cr_w4a8_gemm_ws(xq, xs, q, s, cb, ws, w8, b, acc_out=True)
        torch.cuda.synchronize()
        assert torch.equal(a1, a2) and torch.equal(o1, o2)
        assert torch.equal(w8, cr.cr_w4a8_decode_int8(q, s, cb))


def test_workspace_variants_reject_a_missing_workspace():
    L = cr.lib()
    a = torch.empty(1024, dtype=torch.uint8, device="cuda")
    p = a.data_ptr()
    assert L.cr_w4a8_gemm_ws(p, p, p, p, p, p, None, 16, 16, 256, 0, p, None, None, None) == cr.CR_ERR_INVALID_ARG
    assert L.cr_w4a8_gemm_ws(p, p, p, p, p, p, None, 16, 16, 256, 0, p, None, p + 8, None) == cr.CR_ERR_ALIGNMENT
    assert L.cr_w4a8_linear_ws(p, p, p, p, p, None, 16, 16, 256, 127, 0, p, p, p, None, None) == cr.CR_ERR_INVALID_ARG
    assert L.cr_w4a8_ste_backward_ws(p, p, p, p, p, 4, 16, 256, p, None, None) == cr.CR_ERR_INVALID_ARG
    # empty problems need no workspace
    assert L.cr_w4a8_gemm_ws(p, p, p, p, p, p, None, 0, 16, 256, 0, p, None, None, None) == cr.CR_OK


@pytest.mark.parametrize("M,N,K", [(64, 512, 1024), (1100, 256, 8192)])
def test_ste_backward_ws_equals_pool_call(M, N, K):
    layer = inputs.layer(N, K, 5 * N + K)
    q, s, cb, ws = dev(layer.qdata), dev(layer.srel), dev(layer.codebook), dev(layer.s_channel)
    g = torch.randn(M, N, generator=torch.Generator().manual_seed(M)).to(torch.bfloat16).cuda()
    dx1 = cr.cr_w4a8_ste_backward(g, q, s, cb, ws)
    wt = torch.empty(K, N, dtype=torch.bfloat16, device="cuda")
    dx2 = cr.cr_w4a8_ste_backward_ws(g, q, s, cb, ws, wt)
    torch.cuda.synchronize()
    assert torch.equal(dx1, dx2)
    assert torch.equal(wt, cr.cr_w4a8_dequant_t_bf16(q, s, cb, ws))


# ---------------------------------------------------------------- current device

@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2, reason="needs two GPUs")
def test_calls_on_a_device_that_is_not_current():
    """The binding makes the tensors' device current for the call."""
    M, N, K = 4, 512, 1024
    layer = inputs.layer(N, K, 9)
    x_np = inputs.activations(M, K, 9)
    with torch.cuda.device(0):
        ref = cr.cr_w4a8_linear(bf16_dev(x_np), dev(layer.qdata), dev(layer.srel), dev(layer.codebook),
                                dev(layer.s_channel))
    d1 = torch.device("cuda", 1)
    t = [torch.from_numpy(a).to(d1) for a in (layer.qdata, layer.srel, layer.codebook, layer.s_channel)]
    x1 = torch.from_numpy(x_np.view(np.int16)).to(d1).view(torch.bfloat16)
    with torch.cuda.device(0):
        y = cr.cr_w4a8_linear(x1, *t)
        y2 = cr.cr_w4a8_linear_decode_noalloc(x1, *t)
        with pytest.raises(ValueError):
            cr.cr_w4a8_linear(x1, dev(layer.qdata), *t[1:])
    torch.cuda.synchronize(0)
    torch.cuda.synchronize(1)
    assert torch.equal(y.cpu(), ref.cpu()) and torch.equal(y2.cpu(), ref.cpu())


# ---------------------------------------------------------------- decode GEMV: both weight decodes

def _codebook(kind):
    if kind == "fixed":
        return inputs.codebook()
    if kind == "arange":
        return np.arange(-8, 8, dtype=np.float32)
    if kind == "wide":
        return np.linspace(-300.0, 300.0, 16).astype(np.float32)
    return np.array([3, -1, 0.5, 7, -6, 2, -0.25, 5, -3, 1, -7, 4, 0, -5, 6, -2], np.float32)  # unsorted


@pytest.mark.parametrize("cb_kind", ["fixed", "arange", "wide", "unsorted"])
@pytest.mark.parametrize("scales", ["all_bytes", "generator", "one_large"])
def test_gemv_decodes_every_scale_byte(cb_kind, scales):
    """The decode GEMV picks, per CTA, a split table decode (two byte
    permutes whose int8 results add up to the level inside the MMA) when every
    scale byte of its tiles allows it, and the general decode otherwise.  Both
    must give the oracle's int32 sums and outputs bit for bit: every scale
    byte (NaN and negative ones included), codebooks that saturate or are not
    sorted, and a layer whose scales are ordinary except one large byte in
    one row (so CTAs differ in the decode they take)."""
    M, N, K, seed = 5, 4096 + 48, 2048, 77
    layer = inputs.layer(N, K, seed)
    cb = _codebook(cb_kind)
    srel = layer.srel.copy()
    rng = np.random.default_rng(seed)
    if scales == "all_bytes":
        srel = rng.integers(0, 256, size=srel.shape, dtype=np.uint8)
        srel[:2, :] = np.arange(256, dtype=np.uint8).reshape(2, 128)  # every byte, in two rows
    elif scales == "one_large":
        srel[1000, 7] = 0x7E  # 448: saturates the top levels of the fixed codebook
    x = inputs.activations(M, K, seed)
    ref = oracle.linear(x, layer.qdata, srel, cb, layer.s_channel, threads=8)
    xq, xs = oracle.rotate_quant_act(x, oracle.mp_for(M))
    q, s, c, ws = dev(layer.qdata), dev(srel), dev(cb), dev(layer.s_channel)
    out, acc = cr.cr_w4a8_gemv(dev(xq), dev(xs), q, s, c, ws, m=M, acc_out=True)
    torch.cuda.synchronize()
    assert np.array_equal(host(acc), ref["acc"])
    assert np.array_equal(host(out), ref["y"])
    # the same through the prefill path (GEMV and GEMM agree bit for bit)
    out2 = cr.cr_w4a8_gemm(dev(xq[:M]), dev(xs[:M]), q, s, c, ws)
    torch.cuda.synchronize()
    assert np.array_equal(host(out2), host(out))


@pytest.mark.parametrize("cb_kind", ["fixed", "arange", "unsorted"])
@pytest.mark.parametrize("scales", ["all_bytes", "generator", "one_large"])
@pytest.mark.parametrize("N", [4096 + 48, 4752, 19200])
def test_prepared_layer_decode_matches_oracle(cb_kind, scales, N):
    """A prepared layer (W4A8Linear) checks its scale bytes once and then
    decodes with split tables when all of them have one and each CTA has at
    most two row tiles: N = 4144 (16-row tiles) and N = 4752 (32-row tiles,
    the last one ragged); at N = 19200 (600 tiles of 32 rows) CTAs have more
    and the plain tables serve.  Its forward and its GEMV on quantised
    activations must equal the oracle and the unprepared GEMV bit for bit,
    for layers whose bytes all allow the split form, none do, or all but
    one."""
    K, seed = 2048, 91
    layer = inputs.layer(N, K, seed)
    cb = _codebook(cb_kind)
    srel = layer.srel.copy()
    rng = np.random.default_rng(seed)
    if scales == "all_bytes":
        srel = rng.integers(0, 256, size=srel.shape, dtype=np.uint8)
    elif scales == "one_large":
        srel[N // 2, 3] = 0x7E
    q, s, c, ws = dev(layer.qdata), dev(srel), dev(cb), dev(layer.s_channel)
    lin = cr.W4A8Linear(q, s, c, ws)
    for M in (1, 5, 8):
        x = inputs.activations(M, K, seed + M)
        ref = oracle.linear(x, layer.qdata, srel, cb, layer.s_channel, threads=8)
        y = lin(bf16_dev(x))
        xq, xs = cr.cr_rotate_quant_act(bf16_dev(x), cr.gemv_rows(M))
        y2 = lin.gemv(xq, xs, m=M)
        y3 = cr.cr_w4a8_gemv(xq, xs, q, s, c, ws, m=M)
        torch.cuda.synchronize()
        assert np.array_equal(host(y), ref["y"]), (M, cb_kind, scales)
        assert torch.equal(y2, y3) and torch.equal(y, y2)


def test_int8_rate_kernel_runs_and_counts_its_operations():
    """The INT8 tensor-core rate kernel (the prefill roofline's denominator):
    one launch per SM pair of `iters` groups of four 256 x 256 x 32 MMAs on
    resident operands; it reports 2 * 256 * 256 * 128 * iters operations per
    pair, completes without a device error, and its rate is a plausible
    fraction of the part's dense INT8 figure."""
    pairs = torch.cuda.get_device_properties(0).multi_processor_count // 2
    stream = torch.cuda.current_stream()
    ops = cr.cr_mma_i8_peak(64, stream=stream)
    assert ops == 2.0 * 256 * 256 * 128 * 64 * pairs
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    ops = cr.cr_mma_i8_peak(2048, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    cr.cr_check_device_error()
    tops = ops / (e0.elapsed_time(e1) * 1e-3) / 1e12
    assert 500.0 < tops < 9000.0, tops

