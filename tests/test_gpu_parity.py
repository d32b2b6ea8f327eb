"""GPU parity: every entry point of the C ABI against the CPU oracle, element
by element, on seeded inputs.  Integer stages (unpack/decode, int8
activations, scales, int32 accumulators) must be bit-exact; outputs meet the
normwise tolerance and are also checked bit for bit."""
import os

import numpy as np
import pytest
import torch

import oracle
import w4a8_codebook_quantized_b200 as cr
from w4a8_codebook_quantized_b200 import inputs

from gpu_util import Guarded, assert_output_close, assert_swiglu_close, bf16_dev, dev, host

pytestmark = pytest.mark.gpu

THREADS = max(1, min(32, os.cpu_count() or 1))


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cr.lib()
    yield
    cr.cr_check_device_error()


def _layer_dev(layer):
    return (dev(layer.qdata), dev(layer.srel), dev(layer.codebook), dev(layer.s_channel),
            None if layer.bias is None else dev(layer.bias))


# ---------------------------------------------------------------- decode

def test_decode_exhaustive_scale_bytes_and_codes():
    """All 256 scale bytes x 16 codes (NaN bytes included) through the kernel."""
    N, K = 256, 256
    q = np.tile(np.array([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE], np.uint8), (N, K // 16))
    s = np.repeat(np.arange(256, dtype=np.uint8)[:, None], K // 16, axis=1)
    for cb in (inputs.codebook(), np.arange(-8, 8, dtype=np.float32),
               np.linspace(-300, 300, 16).astype(np.float32)):
        w8 = cr.cr_w4a8_decode_int8(dev(q), dev(s), dev(cb))
        assert np.array_equal(host(w8), oracle.decode_w8(q, s, cb))


@pytest.mark.parametrize("N,K,seed", [(1, 256, 0), (37, 512, 1), (1000, 1024, 2), (4096, 4096, 3)])
def test_decode_random_layers(N, K, seed):
    layer = inputs.layer(N, K, seed)
    out = Guarded((N, K), torch.int8)
    cr.cr_w4a8_decode_int8(dev(layer.qdata), dev(layer.srel), dev(layer.codebook), w8=out.tensor)
    torch.cuda.synchronize()
    assert out.intact()
    assert np.array_equal(host(out.tensor), oracle.decode_w8(layer.qdata, layer.srel, layer.codebook))


# ---------------------------------------------------------------- rotate + quantise

def _rq_case(M, K, seed, mp=None, qmax=127, dist="outliers"):
    x = inputs.activations(M, K, seed, dist)
    MP = M if mp is None else mp
    xq_g = Guarded((MP, K), torch.int8)
    xs_g = Guarded((MP,), torch.float32)
    cr.cr_rotate_quant_act(bf16_dev(x), MP, qmax, xq=xq_g.tensor, xs=xs_g.tensor)
    torch.cuda.synchronize()
    assert xq_g.intact() and xs_g.intact()
    xq_r, xs_r = oracle.rotate_quant_act(x, MP, qmax)
    assert np.array_equal(host(xs_g.tensor).view(np.uint32), xs_r.view(np.uint32))
    assert np.array_equal(host(xq_g.tensor), xq_r)


@pytest.mark.parametrize("M,K,MP", [(1, 256, 1), (3, 1024, 4), (8, 4096, 8), (5, 4096, 8), (2, 8192, 2),
                                    (4, 12288, 4), (2, 16384, 2), (2, 20480, 2), (1, 65536, 1), (33, 768, 33),
                                    (100, 256, 100), (40, 1280, 40), (24, 12288, 24), (17, 16384, 17),
                                    (20, 24576, 20), (18, 32768, 18), (17, 40960, 17), (300, 4096, 300)])
def test_rotate_quant_shapes(M, K, MP):
    """Short batches (at most 16 rows: one block per half-warp) and longer
    ones (a pair of blocks per half-warp in packed fp32x2), across every CTA
    size and register-holding depth of both forms: a lone last block (odd
    K / 256), 64 to 512 threads, two pairs per half-warp, the recomputing
    second pass, and rows beyond one wave of CTAs."""
    _rq_case(M, K, seed=M * 1000 + K, mp=MP)


def test_rotate_quant_other_qmax_and_gelu_inputs():
    _rq_case(6, 2048, 7, qmax=7)
    _rq_case(4, 12288, 8, dist="gelu")
    _rq_case(40, 2048, 9, qmax=7)
    _rq_case(64, 12288, 10, dist="gelu")


@pytest.mark.parametrize("reps,K", [(1, 512), (4, 512), (4, 768)])
def test_rotate_quant_degenerate_rows(reps, K):
    """Zero rows (scale 1), subnormal-only rows, huge rows, a one-hot row; as a
    short batch (5 rows, padded to 8) and as 20-row batches (the packed form,
    with a lone last block when K = 768)."""
    rows = np.zeros((5, K), np.float64)
    rows[1, :7] = 2.0 ** -130
    rows[2] = np.linspace(-2.0 ** 100, 2.0 ** 100, K)
    rows[3, 300] = -1.0
    rows[4] = 1.0
    rows = np.tile(rows, (reps, 1))
    mp = 8 if reps == 1 else rows.shape[0]
    x = torch.from_numpy(rows).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    xq, xs = cr.cr_rotate_quant_act(bf16_dev(x), mp, 127)
    xq_r, xs_r = oracle.rotate_quant_act(x, mp, 127)
    assert np.array_equal(host(xs).view(np.uint32), xs_r.view(np.uint32))
    assert np.array_equal(host(xq), xq_r)
    assert host(xs)[0] == 1.0 and (host(xq)[0] == 0).all()


# ---------------------------------------------------------------- epilogue

@pytest.mark.parametrize("M,N,with_bias,kind", [(1, 8, False, "bf16"), (7, 1000, True, "bf16"),
                                                (64, 4096, False, "f32"), (3, 37, True, "f32"),
                                                (5, 6, True, "bf16")])
def test_epilogue(M, N, with_bias, kind):
    rng = np.random.default_rng(M * N)
    acc = rng.integers(-2 ** 28, 2 ** 28, size=(M, N)).astype(np.int32)
    acc[0, 0] = 16777217
    xs = rng.uniform(1e-3, 0.2, size=M).astype(np.float32)
    ws = rng.uniform(1e-4, 5e-4, size=N).astype(np.float32)
    bias = rng.normal(size=N).astype(np.float32) if with_bias else None
    dt = torch.bfloat16 if kind == "bf16" else torch.float32
    out = Guarded((M, N), dt)
    cr.cr_epilogue(dev(acc), dev(xs), dev(ws), None if bias is None else dev(bias), out=out.tensor)
    torch.cuda.synchronize()
    assert out.intact()
    assert_output_close(host(out.tensor), oracle.epilogue(acc, xs, ws, bias, kind), kind)


# ---------------------------------------------------------------- contraction

def _contraction_case(fn, M, N, K, seed, kind="bf16", with_bias=False, dist="outliers"):
    layer = inputs.layer(N, K, seed, with_bias=with_bias)
    x = inputs.activations(M, K, seed, dist)
    xq_r, xs_r = oracle.rotate_quant_act(x, None, 127)
    w8 = oracle.decode_w8(layer.qdata, layer.srel, layer.codebook)
    acc_r = oracle.gemm_s32(xq_r, w8, THREADS)
    y_r = oracle.epilogue(acc_r, xs_r, layer.s_channel, layer.bias, kind)
    q, s, cb, ws, b = _layer_dev(layer)
    dt = torch.bfloat16 if kind == "bf16" else torch.float32
    out = Guarded((M, N), dt)
    acc = Guarded((M, N), torch.int32)
    fn(dev(xq_r), dev(xs_r), q, s, cb, ws, b, out=out.tensor, acc_out=acc.tensor)
    torch.cuda.synchronize()
    assert out.intact() and acc.intact()
    assert np.array_equal(host(acc.tensor), acc_r)
    assert_output_close(host(out.tensor), y_r, kind)
    # and without the optional accumulator output
    out2 = fn(dev(xq_r), dev(xs_r), q, s, cb, ws, b, out_dtype=dt)
    assert np.array_equal(host(out2), host(out.tensor))
    return host(acc.tensor), host(out.tensor)


@pytest.mark.parametrize("M,N,K", [(1, 16, 256), (1, 1024, 1024), (2, 1000, 512), (3, 17, 768), (4, 4096, 1024),
                                   (8, 4096, 4096), (5, 2048, 2048), (8, 256, 12288), (6, 33, 8192),
                                   (7, 3000, 16384), (2, 520, 20480)])
def test_gemv(M, N, K):
    """Ragged N, every M, K from one stage (1024 columns) up to twenty: the
    activations stream through the ring with the weights, one 1024-column
    chunk per stage."""
    _contraction_case(cr.cr_w4a8_gemv, M, N, K, seed=M + N + K)


@pytest.mark.parametrize("M,N,K", [(8, 8192, 8192), (3, 6000, 2048), (1, 5000, 256), (8, 12288, 4096),
                                   (5, 4752, 7936), (4, 4739, 1280), (8, 4736, 2304), (2, 19200, 1024)])
def test_gemv_several_tiles_per_cta(M, N, K):
    """Layers of at least one 32-row tile per SM (N >= 32 x 148), which take
    32-row tiles: ragged last tiles (N = 4752, 5000, 6000, and 4739, whose
    outputs leave one by one), exactly one tile per SM (N = 4736), CTAs
    walking several tiles with their rings running across tile boundaries
    (chunk counts 1 to 8)."""
    _contraction_case(cr.cr_w4a8_gemv, M, N, K, seed=M + N + K)


@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (8, 256, 512), (100, 300, 1024), (128, 256, 256),
                                   (129, 257, 256), (300, 1000, 1024), (256, 4096, 2048), (2048, 512, 4096),
                                   (17, 17, 768), (640, 1536, 1280)])
def test_gemm(M, N, K):
    _contraction_case(cr.cr_w4a8_gemm, M, N, K, seed=M + N + K)


@pytest.mark.parametrize("M,N,K", [(2048, 4096, 512), (2000, 4000, 768), (4096, 2560, 256), (1100, 9000, 256),
                                   (4352, 2304, 512), (512, 18944, 256), (2048, 4096, 2048)])
def test_gemm_cta_pairs(M, N, K):
    """Shapes with at least one 256 x 256 tile per SM pair take the CTA-pair
    tcgen05 kernel (M = 256 per pair); ragged M and N included, partial last
    waves, and 512 x 18944 = 148 tiles, two whole waves on 74 pairs."""
    _contraction_case(cr.cr_w4a8_gemm, M, N, K, seed=M + N + K, with_bias=(K == 768))


@pytest.mark.parametrize("M,N,K", [(100, 300, 1024), (2048, 4096, 512), (129, 257, 256)])
def test_gemm_s8_on_a_decoded_weight(M, N, K):
    """The contraction on an int8 weight decoded beforehand equals
    cr_w4a8_gemm on the packed layer bit for bit (1-CTA and CTA-pair tiles)."""
    layer = inputs.layer(N, K, M + 3 * N, with_bias=True)
    q, s, cb, ws, b = _layer_dev(layer)
    x = bf16_dev(inputs.activations(M, K, M + 1))
    xq, xs = cr.cr_rotate_quant_act(x)
    w8 = cr.cr_w4a8_decode_int8(q, s, cb)
    o1, a1 = cr.cr_gemm_s8(xq, xs, w8, ws, b, acc_out=True)
    o2, a2 = cr.cr_w4a8_gemm(xq, xs, q, s, cb, ws, b, acc_out=True)
    assert torch.equal(a1, a2) and torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    o3 = cr.cr_gemm_s8(xq, xs, w8, ws, b)  # the TMA-store epilogue path
    assert torch.equal(o3.view(torch.int16), o2.view(torch.int16))


@pytest.mark.parametrize("kind,with_bias", [("f32", False), ("f32", True), ("bf16", True)])
def test_output_kinds_and_bias(kind, with_bias):
    _contraction_case(cr.cr_w4a8_gemv, 3, 520, 1024, 11, kind, with_bias)
    _contraction_case(cr.cr_w4a8_gemm, 200, 520, 1024, 12, kind, with_bias)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 6, 7, 8])
def test_gemv_equals_gemm_bitwise(M):
    """The pages call the decode GEMV bit-identical to the _int_mm path."""
    N, K = 768, 2048
    layer = inputs.layer(N, K, 40 + M)
    x = bf16_dev(inputs.activations(M, K, 40 + M))
    xq, xs = cr.cr_rotate_quant_act(x, cr.gemv_rows(M), 127)
    q, s, cb, ws, b = _layer_dev(layer)
    o1, a1 = cr.cr_w4a8_gemv(xq, xs, q, s, cb, ws, m=M, acc_out=True)
    o2, a2 = cr.cr_w4a8_gemm(xq, xs, q, s, cb, ws, m=M, acc_out=True)
    assert torch.equal(a1, a2) and torch.equal(o1.view(torch.int16), o2.view(torch.int16))


@pytest.mark.parametrize("M,N,K", [(1, 512, 1024), (8, 1024, 4096), (5, 300, 512), (96, 640, 2048)])
def test_linear_end_to_end(M, N, K):
    layer = inputs.layer(N, K, 7 * M)
    x = inputs.activations(M, K, 7 * M)
    ref = oracle.linear(x, layer.qdata, layer.srel, layer.codebook, layer.s_channel, threads=THREADS)
    q, s, cb, ws, b = _layer_dev(layer)
    y = cr.cr_w4a8_linear(bf16_dev(x), q, s, cb, ws)
    assert_output_close(host(y), ref["y"], "bf16")


def test_empty_problems_launch_nothing():
    layer = inputs.layer(16, 256, 1)
    q, s, cb, ws, b = _layer_dev(layer)
    xq = torch.empty(0, 256, dtype=torch.int8, device="cuda")
    xs = torch.empty(0, dtype=torch.float32, device="cuda")
    assert cr.cr_w4a8_gemm(xq, xs, q, s, cb, ws).shape == (0, 16)
    assert cr.cr_w4a8_gemv(xq, xs, q, s, cb, ws).shape == (0, 16)


def test_no_device_error_pending():
    cr.cr_check_device_error()


def test_gemv_back_to_back_and_two_streams():
    """Chained launches (each may start before the previous one ends) and
    launches in flight on two streams at once give the oracle's outputs;
    runs that share a row tile hand their partial sums over exactly."""
    cases = [(8, 4096, 4096, 61), (3, 2000, 1280, 62), (1, 8192, 2048, 63)]
    ref, dev_in = [], []
    for M, N, K, seed in cases:
        layer = inputs.layer(N, K, seed)
        x = inputs.activations(M, K, seed)
        xq_r, xs_r = oracle.rotate_quant_act(x, cr.gemv_rows(M), 127)
        w8 = oracle.decode_w8(layer.qdata, layer.srel, layer.codebook)
        acc_r = oracle.gemm_s32(xq_r[:M], w8, THREADS)
        ref.append(acc_r)
        dev_in.append((dev(xq_r), dev(xs_r)) + _layer_dev(layer) + (M,))
    # back to back on one stream, the same buffers every time
    for (xq, xs, q, s, cb, ws, b, M), acc_r in zip(dev_in, ref):
        outs = [cr.cr_w4a8_gemv(xq, xs, q, s, cb, ws, m=M, acc_out=True)[1] for _ in range(6)]
        for a in outs:
            assert np.array_equal(host(a), acc_r)
    # interleaved on two streams
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    got = []
    for rep in range(4):
        for i, (xq, xs, q, s, cb, ws, b, M) in enumerate(dev_in):
            st = streams[(i + rep) % 2]
            with torch.cuda.stream(st):
                got.append((i, cr.cr_w4a8_gemv(xq, xs, q, s, cb, ws, m=M, acc_out=True)[1]))
    torch.cuda.synchronize()
    for i, a in got:
        assert np.array_equal(host(a), ref[i])


@pytest.mark.parametrize("M", [3, 300])
def test_w4a8_linear_layer_object(M):
    """The prepared layer gives cr_w4a8_linear's outputs bit for bit and checks
    its per-call arguments."""
    N, K = 520, 1024
    layer = inputs.layer(N, K, 90 + M, with_bias=True)
    x = bf16_dev(inputs.activations(M, K, 90 + M))
    q, s, cb, ws, b = _layer_dev(layer)
    lin = cr.W4A8Linear(q, s, cb, ws, b)
    y1 = lin(x)
    y2 = cr.cr_w4a8_linear(x, q, s, cb, ws, b)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    with pytest.raises(ValueError):
        lin(bf16_dev(inputs.activations(M, 512, 1)))
    with pytest.raises(ValueError):
        lin(x, xq_work=torch.empty(cr.gemv_rows(M) if M <= 8 else M, K, dtype=torch.int8))  # host tensor
    # through host buffers: copy in, forward, copy out on one stream, with
    # new contents in the same host buffer on the last call
    x_host = x.cpu().pin_memory()
    out_host = torch.empty(M, N, dtype=torch.bfloat16).pin_memory()
    x_dev, out_dev = torch.empty_like(x), torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    for rep in range(3):
        if rep == 2:
            x2 = bf16_dev(inputs.activations(M, K, 190 + M))
            x_host.copy_(x2.cpu())
            y2 = cr.cr_w4a8_linear(x2, q, s, cb, ws, b)
        out_host.zero_()
        lin.forward_host(x_host, out_host, x_dev, out_dev)
        torch.cuda.synchronize()
        assert torch.equal(out_host.view(torch.int16), y2.cpu().view(torch.int16)), rep


@pytest.mark.parametrize("bound", [False, True])
@pytest.mark.parametrize("pinned,out_kind", [(True, "bf16"), (True, "f32"), (False, "bf16")])
@pytest.mark.parametrize("M,N,K", [(8, 4096, 4096), (5, 776, 2048), (1, 16, 256), (64, 1032, 512), (3, 520, 1024)])
def test_forward_host_copy_paths(bound, pinned, out_kind, M, N, K):
    """Host-buffer forwards over both copy paths: mapped page-locked buffers
    of at most 1 MiB (16-byte multiples) are copied by the library's kernel,
    pageable ones and ragged sizes (3 x 520 bf16) by the copy engine; with
    caller-owned work buffers the layer binds the call once
    (cr_w4a8_plan_bind_host) and then only runs it.  Every call gives
    cr_w4a8_linear's output bit for bit, over repeated calls with the host
    input rewritten in between.  A decode batch with bf16 outputs, N a
    multiple of 8 and a mapped out_host has its GEMV store y there directly
    and leaves out_dev unwritten; every other call leaves y in out_dev too."""
    odt = torch.float32 if out_kind == "f32" else torch.bfloat16
    layer = inputs.layer(N, K, 7 * M + N, with_bias=True)
    q, s, cb, ws, b = _layer_dev(layer)
    lin = cr.W4A8Linear(q, s, cb, ws, b, out_dtype=odt)
    x_host = torch.empty(M, K, dtype=torch.bfloat16)
    out_host = torch.empty(M, N, dtype=odt)
    if pinned:
        x_host, out_host = x_host.pin_memory(), out_host.pin_memory()
    x_dev = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    out_dev = torch.empty(M, N, dtype=odt, device="cuda")
    rows = cr.gemv_rows(M) if M <= 8 else M
    work = (torch.empty(rows, K, dtype=torch.int8, device="cuda"), torch.empty(rows, device="cuda")) if bound \
        else (None, None)
    for rep in range(3):
        x = bf16_dev(inputs.activations(M, K, 500 + 11 * rep + M))
        x_host.copy_(x.cpu())
        ref = cr.cr_w4a8_linear(x, q, s, cb, ws, b, out_dtype=odt)
        out_host.fill_(float("nan"))
        out_dev.fill_(float("nan"))
        lin.forward_host(x_host, out_host, x_dev, out_dev, *work)
        assert (lin._host_args is not None) == bound
        torch.cuda.synchronize()
        view = torch.int32 if odt == torch.float32 else torch.int16
        assert torch.equal(out_host.view(view), ref.cpu().view(view)), rep
        if pinned and M <= 8 and odt == torch.bfloat16 and N % 8 == 0:
            assert bool(torch.isnan(out_dev).all()), rep
        else:
            assert torch.equal(out_dev.view(view), ref.view(view)), rep


def test_plan_reencodes_the_activation_map_when_buffers_change():
    """A prepared layer re-encodes its cached activation map whenever the work
    buffer or M changes: alternating two work buffers and several M on one
    layer gives every call the output of a fresh cr_w4a8_linear."""
    N, K = 1000, 2048
    layer = inputs.layer(N, K, 95)
    q, s, cb, ws, _ = _layer_dev(layer)
    lin = cr.W4A8Linear(q, s, cb, ws)
    works = [(torch.empty(8, K, dtype=torch.int8, device="cuda"), torch.empty(8, device="cuda")) for _ in range(2)]
    for i, M in enumerate([1, 8, 8, 3, 5, 2, 8, 1, 7]):
        x = bf16_dev(inputs.activations(M, K, 200 + i))
        xq, xs = works[i % 2] if i < 6 else works[0]
        y = lin(x, xq_work=xq, xs_work=xs)
        ref = cr.cr_w4a8_linear(x, q, s, cb, ws)
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16)), (i, M)
    f32 = cr.W4A8Linear(q, s, cb, ws, out_dtype=torch.float32)
    x = bf16_dev(inputs.activations(4, K, 300))
    assert torch.equal(f32(x), cr.cr_w4a8_linear(x, q, s, cb, ws, out_dtype=torch.float32))


# ---------------------------------------------------------------- grouped decode (several layers, one input)

@pytest.mark.parametrize("M,K,Ns,bias", [(1, 1024, (512, 512, 512), False),      # q/k/v
                                         (4, 2048, (2048, 512, 512), True),      # q and grouped k/v
                                         (8, 1024, (2816, 2816), False),          # gate/up
                                         (3, 768, (17, 0, 1000, 8), True),        # ragged and an empty layer
                                         (2, 16384, (520, 1040), False)])         # activations streamed
def test_gemv_grouped_matches_oracle_and_single_layers(M, K, Ns, bias):
    """Each layer of a grouped call equals the oracle's contraction of that
    layer (int32 bit-exact, bf16 within tolerance) and the single-layer
    decode GEMV bit for bit."""
    x = inputs.activations(M, K, 300 + M)
    xq_r, xs_r = oracle.rotate_quant_act(x, None, 127)
    xq, xs = dev(xq_r), dev(xs_r)
    layers = [inputs.layer(N, K, 310 + i, with_bias=bias) if N else None for i, N in enumerate(Ns)]
    cb = dev(inputs.codebook())
    specs, guards = [], []
    for ly, N in zip(layers, Ns):
        if ly is None:
            z = torch.empty(0, K // 2, dtype=torch.uint8, device="cuda")
            specs.append((z, torch.empty(0, K // 16, dtype=torch.uint8, device="cuda"),
                          torch.empty(0, device="cuda")))
        else:
            q, s, _, ws, b = _layer_dev(ly)
            specs.append((q, s, ws, b))
        guards.append(Guarded((M, N), torch.bfloat16))
    outs, accs = cr.cr_w4a8_gemv_grouped(xq, xs, cb, specs, outs=[g.tensor for g in guards], acc_out=True)
    torch.cuda.synchronize()
    for (ly, N), go, acc, out in zip(zip(layers, Ns), guards, accs, outs):
        assert go.intact()
        if ly is None:
            continue
        w8 = oracle.decode_w8(ly.qdata, ly.srel, ly.codebook)
        acc_r = oracle.gemm_s32(xq_r, w8, THREADS)
        y_r = oracle.epilogue(acc_r, xs_r, ly.s_channel, ly.bias, "bf16")
        assert np.array_equal(host(acc), acc_r)
        assert_output_close(host(out), y_r, "bf16")
        q, s, _, ws, b = _layer_dev(ly)
        o1, a1 = cr.cr_w4a8_gemv(xq, xs, q, s, cb, ws, b, acc_out=True)
        assert torch.equal(a1, acc) and torch.equal(o1.view(torch.int16), out.view(torch.int16))


@pytest.mark.parametrize("M", [2, 7, 200])
def test_linear_grouped_end_to_end(M):
    """One rotate + quantise for all layers, then the grouped GEMV (M <= 8)
    or a GEMM per layer; each output equals the single-layer forward."""
    K, Ns = 1024, (768, 256, 256)
    x = inputs.activations(M, K, 400 + M)
    cb = dev(inputs.codebook())
    layers = [inputs.layer(N, K, 410 + i, with_bias=(i == 0)) for i, N in enumerate(Ns)]
    devs = [_layer_dev(ly) for ly in layers]
    xd = bf16_dev(x)
    outs = cr.cr_w4a8_linear_grouped(xd, cb, [(q, s, ws, b) for q, s, _, ws, b in devs])
    for ly, (q, s, _, ws, b), y in zip(layers, devs, outs):
        y1 = cr.cr_w4a8_linear(xd, q, s, cb, ws, b)
        assert torch.equal(y1.view(torch.int16), y.view(torch.int16))
        ref = oracle.linear(x, ly.qdata, ly.srel, ly.codebook, ly.s_channel, ly.bias, threads=THREADS)
        assert_output_close(host(y), ref["y"], "bf16")
    # fp32 outputs through the same call
    outs32 = cr.cr_w4a8_linear_grouped(xd, cb, [(q, s, ws, b) for q, s, _, ws, b in devs], out_dtype=torch.float32)
    for ly, y in zip(layers, outs32):
        ref = oracle.linear(x, ly.qdata, ly.srel, ly.codebook, ly.s_channel, ly.bias, out="f32", threads=THREADS)
        assert_output_close(host(y), ref["y"], "f32")


# ---------------------------------------------------------------- SwiGLU on interleaved gate/up rows

def test_interleave_rows_matches_oracle():
    """Bit-exact row interleave for 16-byte, 4-byte and 1-byte row units."""
    rng = np.random.default_rng(9)
    for shape, dtype in (((64, 512), np.uint8), ((2, 16), np.uint8), ((1000,), np.float32), ((6, 3), np.uint8),
                         ((4, 2, 5), np.int16)):
        a = rng.integers(0, 255, size=shape).astype(dtype) if dtype != np.float32 else \
            rng.standard_normal(shape).astype(dtype)
        got = cr.cr_interleave_rows(dev(a))
        assert np.array_equal(host(got), oracle.interleave_rows(a)), (shape, dtype)


def _swiglu_layer(F, K, seed, with_bias=False):
    """An interleaved gate/up layer (numpy) built by the oracle's interleave."""
    g = inputs.layer(F, K, seed, with_bias=with_bias)
    u = inputs.layer(F, K, seed + 1, with_bias=with_bias)
    il = lambda a, b: oracle.interleave_rows(np.concatenate([a, b], axis=0))
    return (il(g.qdata, u.qdata), il(g.srel, u.srel), g.codebook, il(g.s_channel, u.s_channel),
            None if g.bias is None else il(g.bias, u.bias))


def _swiglu_case(fn, M, N, K, seed, kind="bf16", with_bias=False):
    qd, sr, cbk, wsc, bs = _swiglu_layer(N // 2, K, seed, with_bias)
    x = inputs.activations(M, K, seed)
    xq_r, xs_r = oracle.rotate_quant_act(x, None, 127)
    acc_r = oracle.gemm_s32(xq_r, oracle.decode_w8(qd, sr, cbk), THREADS)
    y_r = oracle.epilogue_swiglu(acc_r, xs_r, wsc, bs, kind)
    dt = torch.bfloat16 if kind == "bf16" else torch.float32
    out = Guarded((M, N // 2), dt)
    fn(dev(xq_r), dev(xs_r), dev(qd), dev(sr), dev(cbk), dev(wsc), None if bs is None else dev(bs), out=out.tensor)
    torch.cuda.synchronize()
    assert out.intact()
    assert_swiglu_close(host(out.tensor), y_r, kind)
    return host(out.tensor)


@pytest.mark.parametrize("M,N,K,kind,bias", [(1, 32, 256, "bf16", False), (8, 4096, 1024, "bf16", False),
                                             (3, 26, 512, "bf16", True), (5, 1000, 2048, "f32", True),
                                             (7, 2048, 16384, "bf16", False), (3, 4800, 1024, "bf16", True),
                                             (8, 9000, 2048, "f32", False)])
def test_gemv_swiglu(M, N, K, kind, bias):
    _swiglu_case(cr.cr_w4a8_gemv_swiglu, M, N, K, M + N + K, kind, bias)


@pytest.mark.parametrize("M,N,K,kind,bias", [(100, 512, 512, "bf16", False),     # one-CTA kernel, TMA stores
                                             (129, 26, 256, "bf16", True),       # F = 13: per-thread stores
                                             (300, 1000, 1024, "f32", True),     # F = 500: fp32 TMA stores
                                             (300, 1000, 1024, "bf16", False),   # F = 500: per-thread stores
                                             (2048, 4096, 512, "bf16", True),    # CTA pairs
                                             (2000, 4000, 256, "f32", False)])   # CTA pairs, ragged, fp32
def test_gemm_swiglu(M, N, K, kind, bias):
    _swiglu_case(cr.cr_w4a8_gemm_swiglu, M, N, K, M + N + K, kind, bias)


@pytest.mark.parametrize("M", [1, 2, 5, 8])
def test_gemv_swiglu_equals_gemm_swiglu_bitwise(M):
    N, K = 768, 2048
    qd, sr, cbk, wsc, bs = (None if a is None else dev(a) for a in _swiglu_layer(N // 2, K, 60 + M, True))
    x = bf16_dev(inputs.activations(M, K, 60 + M))
    xq, xs = cr.cr_rotate_quant_act(x, cr.gemv_rows(M), 127)
    for dt in (torch.bfloat16, torch.float32):
        o1 = cr.cr_w4a8_gemv_swiglu(xq, xs, qd, sr, cbk, wsc, bs, m=M, out_dtype=dt)
        o2 = cr.cr_w4a8_gemm_swiglu(xq, xs, qd, sr, cbk, wsc, bs, m=M, out_dtype=dt)
        assert torch.equal(o1.view(torch.int16) if dt == torch.bfloat16 else o1.view(torch.int32),
                           o2.view(torch.int16) if dt == torch.bfloat16 else o2.view(torch.int32))


@pytest.mark.parametrize("M", [4, 300])
def test_linear_swiglu_from_separate_gate_and_up(M):
    """interleave_gate_up on the device from separate gate and up layers,
    then the fused forward: equal to the oracle's SwiGLU forward."""
    F, K = 512, 1024
    g = inputs.layer(F, K, 80, with_bias=True)
    u = inputs.layer(F, K, 81, with_bias=True)
    layer = cr.interleave_gate_up((dev(g.qdata), dev(g.srel), dev(g.s_channel), dev(g.bias)),
                                  (dev(u.qdata), dev(u.srel), dev(u.s_channel), dev(u.bias)))
    x = inputs.activations(M, K, 82)
    cb = dev(g.codebook)
    y = cr.cr_w4a8_linear_swiglu(bf16_dev(x), layer[0], layer[1], cb, layer[2], layer[3])
    il = lambda a, b: oracle.interleave_rows(np.concatenate([a, b], axis=0))
    ref = oracle.linear_swiglu(x, il(g.qdata, u.qdata), il(g.srel, u.srel), g.codebook,
                               il(g.s_channel, u.s_channel), il(g.bias, u.bias), threads=THREADS)
    assert y.shape == (M, F)
    assert_swiglu_close(host(y), ref["y"], "bf16")


# ---------------------------------------------------------------- offline quantiser

def _edge_rows(K):
    """Rows that reach the quantiser's corner cases: an all-zero row (every
    clamp at 1e-8), zero and tiny groups next to normal ones (fp8 zero and
    subnormal s_rel), exact codebook multiples, one-hot groups, a negative
    row and a row of equal values."""
    cb = inputs.codebook()
    rng = np.random.default_rng(21)
    rows = [np.zeros(K)]
    r = rng.standard_normal(K) * 0.02
    r[:16] = 0.0
    r[16:32] *= 1e-4
    r[32:48] *= 1e-7
    rows.append(r)
    rows.append(np.tile(cb, K // 16) * 0.03)
    oh = np.zeros(K)
    oh[::16] = 0.5
    oh[5::16] = -0.01
    rows.append(oh)
    rows.append(-np.abs(rng.standard_normal(K)))
    rows.append(np.full(K, 0.125))
    return np.array(rows, dtype=np.float32)


@pytest.mark.parametrize("N,K", [(1, 16), (3, 48), (37, 512), (300, 4096), (64, 16384), (6, 1024)])
def test_quantize_rotated_bit_exact(N, K):
    w = inputs.rotated_weights(N, K, N + K) if (N, K) != (6, 1024) else _edge_rows(K)
    cb = inputs.codebook()
    q_r, s_r, ch_r = oracle.quantize_rotated(w, cb)
    q, s, ch, _ = cr.cr_w4a8_quantize_rotated(dev(w), dev(cb))
    torch.cuda.synchronize()
    assert np.array_equal(host(s), s_r)
    assert np.array_equal(host(ch).view(np.uint32), ch_r.view(np.uint32))
    assert np.array_equal(host(q), q_r)


def test_quantize_rotated_sampled_rows_full_size():
    """16384 x 16384 on the GPU; rows are independent, so a sample of rows is
    checked against the oracle run on those rows alone."""
    N = K = 16384
    cb = inputs.codebook()
    w = torch.empty(N, K, dtype=torch.float32, device="cuda")
    chunk = 2048
    for r0 in range(0, N, chunk):
        w[r0:r0 + chunk] = dev(inputs.rotated_weights(chunk, K, 1000 + r0))
    q, s, ch, _ = cr.cr_w4a8_quantize_rotated(w, dev(cb))
    torch.cuda.synchronize()
    for r in (0, 1, 2047, 2048, 9000, N - 1):
        wr = host(w[r:r + 1])
        q_r, s_r, ch_r = oracle.quantize_rotated(wr, cb)
        assert np.array_equal(host(q[r:r + 1]), q_r) and np.array_equal(host(s[r:r + 1]), s_r)
        assert np.array_equal(host(ch[r:r + 1]).view(np.uint32), ch_r.view(np.uint32))


@pytest.mark.parametrize("stochastic", [False, True])
def test_assign_codes_bit_exact(stochastic):
    """Codes for updated weights on the stored scales (requantize_codes_),
    deterministic and with uniform draws passed in."""
    N, K = 200, 2048
    cb = inputs.codebook()
    w = inputs.rotated_weights(N, K, 31)
    _, s, ch = oracle.quantize_rotated(w, cb)
    w2 = (w + 0.1 * inputs.rotated_weights(N, K, 32)).astype(np.float32)
    u = inputs.uniforms(N, K, 33) if stochastic else None
    q_r = oracle.assign_codes(w2, s, ch, cb, u)
    q = cr.cr_w4a8_assign_codes(dev(w2), dev(s), dev(ch), dev(cb), None if u is None else dev(u))
    torch.cuda.synchronize()
    assert np.array_equal(host(q), q_r)


def test_quantised_layer_runs_through_the_forward():
    """A layer quantised on the GPU feeds the forward directly, and its output
    equals the oracle forward of the oracle-quantised layer bit for bit."""
    N, K, M = 512, 1024, 4
    cb = inputs.codebook()
    w = inputs.rotated_weights(N, K, 41)
    q, s, ch, cbd = cr.cr_w4a8_quantize_rotated(dev(w), dev(cb))
    x = inputs.activations(M, K, 42)
    y = cr.cr_w4a8_linear(bf16_dev(x), q, s, cbd, ch)
    q_r, s_r, ch_r = oracle.quantize_rotated(w, cb)
    ref = oracle.linear(x, q_r, s_r, cb, ch_r, threads=THREADS)
    assert_output_close(host(y), ref["y"], "bf16")


# ---------------------------------------------------------------- straight-through backward

@pytest.mark.parametrize("N,K", [(8, 256), (520, 1024), (4096, 4096), (200, 2048)])
def test_dequant_t_bf16_bit_exact(N, K):
    layer = inputs.layer(N, K, N + K)
    q, s, cb, ws, _ = _layer_dev(layer)
    wt = cr.cr_w4a8_dequant_t_bf16(q, s, cb, ws)
    torch.cuda.synchronize()
    ref = oracle.dequant_bf16(layer.qdata, layer.srel, layer.codebook, layer.s_channel)
    assert np.array_equal(host(wt), np.ascontiguousarray(ref.T))


@pytest.mark.parametrize("M,N,K", [(1, 8, 256), (64, 512, 1024), (300, 1000, 768), (129, 72, 2048),
                                   (1024, 2048, 1024),
                                   (1100, 256, 8192), (2000, 72, 4096)])  # the last two on CTA pairs
def test_ste_backward(M, N, K):
    """dx against the oracle (double sums, one rounding) and against torch's
    fp32 matmul of the same bf16 operands, elementwise within the bound the
    arithmetic gives: half a bf16 ulp for each side's final rounding plus the
    fp32 accumulation error of a sum of N products, N * 2^-24 * sum|g * w|
    (the pages leave the accumulation order to the matmul); ragged M, N not a
    multiple of 64, K tails of the 256-column tiles."""
    layer = inputs.layer(N, K, 3 * N + K)
    rng = np.random.default_rng(M + N + K)
    g = torch.from_numpy(rng.standard_normal((M, N)).astype(np.float32)).to(torch.bfloat16)
    g_bits = g.view(torch.int16).numpy().view(np.uint16)
    q, s, cb, ws, _ = _layer_dev(layer)
    dx = Guarded((M, K), torch.bfloat16)
    cr.cr_w4a8_ste_backward(g.cuda(), q, s, cb, ws, dx=dx.tensor)
    torch.cuda.synchronize()
    assert dx.intact()
    got = host(dx.tensor)
    ref = oracle.ste_backward(g_bits, layer.qdata, layer.srel, layer.codebook, layer.s_channel)
    from gpu_util import bf16_bits_to_f64
    w = torch.from_numpy(oracle.dequant_bf16(layer.qdata, layer.srel, layer.codebook, layer.s_channel)
                         .view(np.int16)).view(torch.bfloat16).float()
    absum = np.abs(g.float().numpy().astype(np.float64)) @ np.abs(w.numpy().astype(np.float64))
    acc = N * 2.0 ** -24 * absum
    gf, rf = bf16_bits_to_f64(got), bf16_bits_to_f64(ref)
    bound = 2.0 ** -8 * (np.abs(gf) + np.abs(rf)) + acc + 1e-30
    assert np.all(np.abs(gf - rf) <= bound), np.max(np.abs(gf - rf) / bound)
    t32 = (g.float() @ w).numpy().astype(np.float64)
    assert np.all(np.abs(gf - t32) <= 2.0 ** -8 * np.abs(gf) + 2 * acc + 1e-30)
    # and most elements agree with the oracle exactly
    assert (got == ref).mean() > 0.9


def test_ste_backward_empty_layer_gives_zero():
    layer = inputs.layer(8, 256, 1)
    q, s, cb, ws, _ = _layer_dev(layer)
    dx = torch.full((4, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    cr.cr_w4a8_ste_backward(torch.empty(4, 0, dtype=torch.bfloat16, device="cuda"), q[:0], s[:0], cb, ws[:0], dx=dx)
    torch.cuda.synchronize()
    assert not dx.float().abs().sum().item()


# ---------------------------------------------------------------- failure detection

def test_bounded_wait_runs_out_and_is_reported():
    """A wait that nothing completes gives up after its limit, the host reads
    CR_ERR_TIMEOUT once (the word is cleared), and the context keeps working."""
    cr.cr_check_device_error()
    cr.cr_selftest_wait_timeout(0.005)
    with pytest.raises(cr.CrError) as err:
        cr.cr_check_device_error()
    assert err.value.status == cr.CR_ERR_TIMEOUT
    cr.cr_check_device_error()  # cleared
    layer = inputs.layer(256, 1024, 7)
    q, s, cb, ws, _ = _layer_dev(layer)
    x = bf16_dev(inputs.activations(4, 1024, 7))
    xq, xs = cr.cr_rotate_quant_act(x, 4)
    o1, a1 = cr.cr_w4a8_gemv(xq, xs, q, s, cb, ws, m=4, acc_out=True)
    o2, a2 = cr.cr_w4a8_gemm(xq, xs, q, s, cb, ws, m=4, acc_out=True)
    cr.cr_check_device_error()
    assert torch.equal(a1, a2)
