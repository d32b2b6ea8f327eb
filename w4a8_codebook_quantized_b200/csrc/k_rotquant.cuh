// k_rotquant.cuh -- block-256 regular-Hadamard rotation of bf16 activation
// rows fused with per-token symmetric int8 quantisation.
//
// What it computes (ai-toolkit convrot_w4a8_quant.py, prepare_act and
// w4a8_act_quant_kernel; h3-rs src/weights.rs, hadamard / rotate_activation):
// each 256-column block of a row is multiplied by H_256 = h4^(x4) / 16, the
// row's absolute maximum gives the scale amax / qmax, and every value is
// rounded to nearest even after the division and clamped to +-qmax.  Rows
// M..MP-1 are the decode GEMV's padding: zeros with scale 1.
//
// fp32 order (the pages leave it open; this order is the layer's definition
// here): the bf16 inputs widen exactly; the four base-4 digits of the index
// within the block are processed in the order stride 1, 4, 16, 64; one
// quadruple (v0, v1, v2, v3) along a digit becomes S - 2 v[3-a] with
// S = (v0 + v1) + (v2 + v3); the result is scaled by 1/16.
//
// Layout: one CTA per row, of 256 threads (512 for short batches of long
// rows, where the few CTAs would otherwise leave most SMs idle).  A half-warp (16 lanes) owns one
// 256-element block, viewed as a 16 x 16 matrix with element 16a + b: lane L
// first holds row a = L (16 contiguous bf16, two 16-byte loads), applies the
// stride-1 and stride-4 digits in registers, transposes through shared memory
// so that it holds column b = L, applies the stride-16 and stride-64 digits in
// registers, and keeps the 16 fp32 results in registers until the row's
// maximum is known.  The quantised bytes go back to row order through a
// second, byte-wide shared-memory transpose and leave as one 16-byte store per
// lane.  HBM traffic is the algorithmic minimum: 2 bytes read and 1 written
// per element.  Rows with K > 4096 * kMaxBlocksInRegs are handled by a
// second pass that recomputes the rotation instead of holding it.
#pragma once

#include "cr_device.cuh"

namespace cr {
namespace rq {

constexpr int kThreads = 256;              // the CTA size for batches of many rows
constexpr int kWideThreads = 512;          // ... and for at most kWideRows rows of K >= 8192
constexpr int kWideRows = 16;
constexpr int kMaxBlocksInRegs = 4;        // per half-warp: K <= 16384 (32768 wide) stays in registers

// One digit of the rotation on a quadruple (row a of h4 is all ones except
// -1 at column 3 - a).  2v is exact, so fma(-2, v, S) is S - 2v rounded once.
__device__ __forceinline__ void h4_quad(float &a0, float &a1, float &a2, float &a3)
{
    const float S = __fadd_rn(__fadd_rn(a0, a1), __fadd_rn(a2, a3));
    const float y0 = __fmaf_rn(-2.0f, a3, S);
    const float y1 = __fmaf_rn(-2.0f, a2, S);
    const float y2 = __fmaf_rn(-2.0f, a1, S);
    const float y3 = __fmaf_rn(-2.0f, a0, S);
    a0 = y0;
    a1 = y1;
    a2 = y2;
    a3 = y3;
}

// Rotate one 256-element block.  On return lane L of the half-warp holds
// v[a] = 16 x rotated element 16a + L (a = 0..15).  `tr` is this half-warp's
// 16 x 16 fp32 transpose buffer (16-byte aligned).
__device__ __forceinline__ void rotate_block(const uint16_t *__restrict__ blk, int L, float *tr, unsigned hmask,
                                             float (&v)[16])
{
    const uint4 *src = reinterpret_cast<const uint4 *>(blk + 16 * L);
    const uint4 p0 = __ldg(src);
    const uint4 p1 = __ldg(src + 1);
    const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);             // element 2i: low half
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);  // element 2i+1: high half
    }
    // stride 1 (digit d0 = b % 4), then stride 4 (digit d1 = b / 4)
#pragma unroll
    for (int q = 0; q < 4; ++q)
        h4_quad(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
#pragma unroll
    for (int q = 0; q < 4; ++q)
        h4_quad(v[q], v[q + 4], v[q + 8], v[q + 12]);
    // Transpose through shared memory: row L goes out as four 16-byte stores,
    // column L comes back as 16 scalar loads.  Chunk c of row a lives at chunk
    // position c ^ ((a >> 1) & 3), which makes both sides conflict-free.
    {
        float4 *rowp = reinterpret_cast<float4 *>(tr + 16 * L);
        const int sw = (L >> 1) & 3;
#pragma unroll
        for (int c = 0; c < 4; ++c)
            rowp[c ^ sw] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
    }
    __syncwarp(hmask);
    {
        const float *base[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
            base[k] = tr + 4 * ((L >> 2) ^ k) + (L & 3);
#pragma unroll
        for (int a = 0; a < 16; ++a)
            v[a] = base[(a >> 1) & 3][16 * a];
    }
    __syncwarp(hmask);
    // stride 16 (digit d2 = a % 4), then stride 64 (digit d3 = a / 4)
#pragma unroll
    for (int q = 0; q < 4; ++q)
        h4_quad(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
#pragma unroll
    for (int q = 0; q < 4; ++q)
        h4_quad(v[q], v[q + 4], v[q + 8], v[q + 12]);
    // The final 1/16 is not applied here: v holds R = 16 r.  Scaling by a power
    // of two commutes with rounding away from subnormals, so the quantiser
    // works on R with the scale multiplied by 16 and gets the same integers
    // (rows whose values reach the subnormal range take an exact path that
    // applies the 1/16 per element).
}

// Quantise this lane's 16 column values of one block and store them in row
// order.  v holds R = 16 r (see rotate_block); scale is s, the row's scale.
//
// Fast path (any row whose max |r| >= 2^-100): q = rint(r / s) without a
// per-element division.  inv16 = (1/s rounded) / 16, so t = R * inv16 equals
// r * (1/s rounded) rounded; it differs from the correctly rounded quotient
// v = r / s by at most 3 * 2^-24 * |r / s| <= 3 * 2^-24 * 128 < 2^-15.  Unless t
// lies within 2^-15 of a half-integer, t and v round to the same integer and
// neither is a tie; those rare elements are redone with the exact quotient
// R / (16 s).  Adding 1.5 * 2^23 rounds t to an integer (nearest even) in the
// low mantissa bits, whose low byte is the two's-complement int8 result.  No
// clamp is needed: |t| <= qmax + 2^-15 cannot round past qmax.
//
// Exact path (a row of tiny values, max |r| < 2^-100): r = R / 16 rounded per
// element (it may be subnormal), q = rint(r / s) with the division, clamped.
__device__ __forceinline__ void quantise_store(const float (&v)[16], float scale, float inv16, int32_t qmax,
                                               bool exact_row, int L, uint8_t *tb, unsigned hmask,
                                               int8_t *__restrict__ dst_block)
{
    const float kMagic = 12582912.0f;  // 1.5 * 2^23
    if (!exact_row) {
        uint32_t near = 0;
#pragma unroll
        for (int a = 0; a < 16; ++a) {
            const float t = __fmul_rn(v[a], inv16);
            const float tm = __fadd_rn(t, kMagic);
            const float d = __fsub_rn(t, __fsub_rn(tm, kMagic));
            near |= (fabsf(d) >= 0.499969482421875f ? 1u : 0u) << a;  // within 2^-15 of k + 1/2
            tb[16 * a + L] = (uint8_t)__float_as_uint(tm);
        }
        if (near) {
            const float s16 = __fmul_rn(scale, 16.0f);
#pragma unroll
            for (int a = 0; a < 16; ++a)
                if ((near >> a) & 1u) {
                    const int32_t q = __float2int_rn(__fdiv_rn(v[a], s16));
                    tb[16 * a + L] = (uint8_t)min(max(q, -qmax), qmax);
                }
        }
    } else {
#pragma unroll
        for (int a = 0; a < 16; ++a) {
            const float r = __fmul_rn(v[a], 0.0625f);
            const int32_t q = __float2int_rn(__fdiv_rn(r, scale));
            tb[16 * a + L] = (uint8_t)min(max(q, -qmax), qmax);
        }
    }
    __syncwarp(hmask);
    const uint4 o = *reinterpret_cast<const uint4 *>(tb + 16 * L);
    *reinterpret_cast<uint4 *>(dst_block + 16 * L) = o;
    __syncwarp(hmask);
}

// max |v[i]| over 16 values as a tree of depth 4 (fmaxf drops NaN operands,
// so the result is NaN-free and >= 0 for any inputs; max is exact in any
// order).
__device__ __forceinline__ float max_abs16(const float (&v)[16])
{
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        m[i] = fmaxf(fabsf(v[i]), fabsf(v[i + 8]));
#pragma unroll
    for (int i = 0; i < 4; ++i)
        m[i] = fmaxf(m[i], m[i + 4]);
    return fmaxf(fmaxf(m[0], m[2]), fmaxf(m[1], m[3]));
}

template <int J, bool kRecompute, int THREADS>
__global__ void __launch_bounds__(THREADS) rotquant_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t K,
                                                            int qmax, int8_t *__restrict__ xq,
                                                            float *__restrict__ xs)
{
    // half-warp buffers 16 floats apart in bank space: the two halves of a warp
    // never touch the same bank in one transpose step
    constexpr int kHalfWarps = THREADS / 16;  // blocks of 256 in flight per CTA
    __shared__ __align__(16) float tr_all[kHalfWarps][16 * 16 + 16];
    __shared__ __align__(16) uint8_t tb_all[kHalfWarps][272];
    __shared__ float warp_max[THREADS / 32];

    // Let a programmatic dependent (the decode GEMV) start its weight stream
    // now; it waits for this grid's results before it reads them.
    asm volatile("griddepcontrol.launch_dependents;" :::);
    // Launched as a programmatic dependent itself, this grid may be resident
    // before the previous kernel on the stream has finished: x may still be
    // in the making and xq / xs still being read, so nothing is read or
    // written before that kernel completes.  Only an L2 prefetch of this
    // CTA's row of x goes out first: the L2 is where the device's writes
    // become visible, so a prefetch cannot make a later load return an old
    // value, and the row's loads after the wait then find it there.
    if (threadIdx.x == 0 && (int64_t)blockIdx.x < M)
        bulk_prefetch_l2(x + (int64_t)blockIdx.x * K, (uint32_t)(K * 2));
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const int tid = threadIdx.x;
    const int hw = tid >> 4, L = tid & 15, warp = tid >> 5, lane = tid & 31;
    const unsigned hmask = 0xFFFFu << (16 * (hw & 1));
    const int64_t m = blockIdx.x;
    const int NB = (int)(K / 256);
    int8_t *__restrict__ qrow = xq + m * K;

    if (m >= M) {  // padding row of the decode GEMV operand
        for (int64_t c = tid; c < K / 16; c += THREADS)
            reinterpret_cast<uint4 *>(qrow)[c] = make_uint4(0u, 0u, 0u, 0u);
        if (tid == 0)
            xs[m] = 1.0f;
        return;
    }

    const uint16_t *__restrict__ xrow = x + m * K;
    float *tr = tr_all[hw];
    uint8_t *tb = tb_all[hw];
    float amax = 0.0f;
    float v[kRecompute ? 1 : J][16];

    if (!kRecompute) {
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int b = hw + kHalfWarps * j;
            if (b < NB) {
                rotate_block(xrow + 256 * b, L, tr, hmask, v[j]);
                amax = fmaxf(amax, max_abs16(v[j]));
            }
        }
    } else {
        for (int b = hw; b < NB; b += kHalfWarps) {
            rotate_block(xrow + 256 * b, L, tr, hmask, v[0]);
            amax = fmaxf(amax, max_abs16(v[0]));
        }
    }

    // row maximum (exact in any order).  amax is >= 0 and never NaN, and
    // such floats order like their bit patterns as unsigned integers: one
    // warp reduction instruction on the bits.
    {
        uint32_t bits = __float_as_uint(amax);
        asm volatile("redux.sync.max.u32 %0, %0, 0xffffffff;" : "+r"(bits));
        amax = __uint_as_float(bits);
    }
    if (lane == 0)
        warp_max[warp] = amax;
    __syncthreads();
    float rmax = warp_max[0];
#pragma unroll
    for (int w = 1; w < THREADS / 32; ++w)
        rmax = fmaxf(rmax, warp_max[w]);
    // rmax is max |R| = 16 max |r|; the row maximum of r is rmax / 16 rounded
    // (rounding is monotonic, so that is also the max of the rounded r).
    const float rowmax = __fmul_rn(rmax, 0.0625f);
    const float scale = (rowmax > 0.0f) ? __fdiv_rn(rowmax, (float)qmax) : 1.0f;
    const bool exact_row = rowmax > 0.0f && rowmax < 7.8886091e-31f;  // max |r| < 2^-100
    const float inv16 = __fmul_rn(__frcp_rn(scale), 0.0625f);

    if (!kRecompute) {
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int b = hw + kHalfWarps * j;
            if (b < NB)
                quantise_store(v[j], scale, inv16, qmax, exact_row, L, tb, hmask, qrow + 256 * b);
        }
    } else {
        for (int b = hw; b < NB; b += kHalfWarps) {
            rotate_block(xrow + 256 * b, L, tr, hmask, v[0]);
            quantise_store(v[0], scale, inv16, qmax, exact_row, L, tb, hmask, qrow + 256 * b);
        }
    }
    if (tid == 0)
        xs[m] = scale;
}

template <int THREADS>
inline cudaError_t launch_t(const uint16_t *x, int64_t M, int64_t K, int64_t MP, int qmax, int8_t *xq, float *xs,
                            cudaStream_t stream)
{
    constexpr int kHalfWarps = THREADS / 16;
    const int64_t per_hw = (K / 256 + kHalfWarps - 1) / kHalfWarps;  // blocks per half-warp
    void (*kern)(const uint16_t *, int64_t, int64_t, int, int8_t *, float *) =
        per_hw <= 1   ? rotquant_kernel<1, false, THREADS>
        : per_hw == 2 ? rotquant_kernel<2, false, THREADS>
        : per_hw == 3 ? rotquant_kernel<3, false, THREADS>
        : per_hw == 4 ? rotquant_kernel<4, false, THREADS>
                      : rotquant_kernel<1, true, THREADS>;
    // a programmatic dependent of the previous kernel on the stream: its
    // launch overlaps that kernel's tail, and the kernel waits for it
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)MP);
    cfg.blockDim = dim3(THREADS);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, x, M, K, qmax, xq, xs);
}

// One CTA per row: 512 threads when there are few rows of K >= 8192 (the
// decode batches), 256 otherwise.
inline cudaError_t launch(const uint16_t *x, int64_t M, int64_t K, int64_t MP, int qmax, int8_t *xq, float *xs,
                          cudaStream_t stream)
{
    if (MP <= kWideRows && K >= 8192)
        return launch_t<kWideThreads>(x, M, K, MP, qmax, xq, xs, stream);
    return launch_t<kThreads>(x, M, K, MP, qmax, xq, xs, stream);
}

}  // namespace rq
}  // namespace cr
