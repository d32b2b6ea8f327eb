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
// Layout: one CTA per row, in one of two forms.  Both view a 256-element
// block as a 16 x 16 matrix with element 16a + b, and both give a block to a
// half-warp (16 lanes): lane L first holds row a = L (16 contiguous bf16, two
// 16-byte loads), applies the stride-1 and stride-4 digits in registers,
// transposes through shared memory so that it holds column b = L, applies the
// stride-16 and stride-64 digits in registers, and keeps the fp32 results in
// registers until the row's maximum is known.  The quantised bytes go back to
// row order through a byte-wide shared-memory transpose and leave as one
// 16-byte store per lane and block.  HBM traffic is the algorithmic minimum:
// 2 bytes read and 1 written per element.
//  - Batches of many rows (prefill): a half-warp owns a PAIR of blocks and
//    computes both at once with the packed fp32x2 arithmetic of sm_100
//    (add / sub / mul / fma .f32x2: each half of a 64-bit register is one fp32
//    value, rounded exactly as the scalar instruction rounds it), so one
//    instruction does the work of two; the scalar form was bound by
//    instruction issue at these sizes, and this halves its arithmetic.
//  - Short batches (decode, at most kShortRows rows): a half-warp owns ONE
//    block in scalar fp32, so that twice as many threads share a row and each
//    one's chain of dependent instructions is shortest: here few CTAs run and
//    the kernel's latency, not its throughput, is what a step waits for.
// Rows too long for the registers are handled by a second pass that
// recomputes the rotation instead of holding it.
#pragma once

#include "cr_device.cuh"

namespace cr {
namespace rq {

constexpr int kShortRows = 16;  // batches of at most this many rows take the scalar form
// Shared memory each short-batch CTA reserves beyond what it uses.  In a
// decode step the rotation's few CTAs become resident while the previous
// GEMV still fills the SMs, and the block scheduler may stack up to four of
// them (512 threads each) on the first SM that frees up, where they share its
// issue slots.  The reservation caps them at two per SM while a GEMV CTA can
// still sit beside one.  Measured on B200: the M = 8, N = K = 8192 decode step
// 15.4 -> 14.2 us, the others unchanged or slightly faster; 80 KB and more
// slowed the M <= 4 steps.
constexpr int kShortReserve = 60 * 1024;

// ================================================================ scalar form (short batches)

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

// One block per half-warp: THREADS / 16 half-warps per row, each holding up
// to J blocks in registers (kRecompute: one at a time, rotating every block
// twice).
template <int J, bool kRecompute, int THREADS>
__global__ void __launch_bounds__(THREADS) rotquant_rows_kernel(const uint16_t *__restrict__ x, int64_t M,
                                                                 int64_t K, int qmax, int8_t *__restrict__ xq,
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
inline cudaError_t launch_rows_t(const uint16_t *x, int64_t M, int64_t K, int64_t MP, int qmax, int8_t *xq,
                                 float *xs, cudaStream_t stream)
{
    constexpr int kHalfWarps = THREADS / 16;
    const int64_t per_hw = (K / 256 + kHalfWarps - 1) / kHalfWarps;  // blocks per half-warp
    void (*kern)(const uint16_t *, int64_t, int64_t, int, int8_t *, float *) =
        per_hw <= 1   ? rotquant_rows_kernel<1, false, THREADS>
        : per_hw == 2 ? rotquant_rows_kernel<2, false, THREADS>
        : per_hw == 3 ? rotquant_rows_kernel<3, false, THREADS>
        : per_hw == 4 ? rotquant_rows_kernel<4, false, THREADS>
                      : rotquant_rows_kernel<1, true, THREADS>;
    // a programmatic dependent of the previous kernel on the stream: its
    // launch overlaps that kernel's tail, and the kernel waits for it
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)MP);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = kShortReserve;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, x, M, K, qmax, xq, xs);
}

// ================================================================ packed form (batches of many rows)

// ---------------------------------------------------------------- fp32 pairs in 64-bit registers

__device__ __forceinline__ uint64_t pk(uint32_t lo, uint32_t hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}

__device__ __forceinline__ void unpk(uint64_t v, uint32_t &lo, uint32_t &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
}

__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// One digit of the rotation on a quadruple of pairs (row a of h4 is all ones
// except -1 at column 3 - a).  2v is exact, so fma(-2, v, S) is S - 2v
// rounded once.
__device__ __forceinline__ void h4_quad2(uint64_t &a0, uint64_t &a1, uint64_t &a2, uint64_t &a3)
{
    const uint64_t m2 = 0xC0000000C0000000ull;  // (-2.0f, -2.0f)
    const uint64_t S = add2(add2(a0, a1), add2(a2, a3));
    const uint64_t y0 = fma2(m2, a3, S);
    const uint64_t y1 = fma2(m2, a2, S);
    const uint64_t y2 = fma2(m2, a1, S);
    const uint64_t y3 = fma2(m2, a0, S);
    a0 = y0;
    a1 = y1;
    a2 = y2;
    a3 = y3;
}

// Rotate a pair of 256-element blocks: blk0 into the low halves, blk1 into
// the high halves (blk1 == nullptr stands for a block of zeros).  On return
// lane L of the half-warp holds v[a] = 16 x rotated element 16a + L of both
// blocks (a = 0..15).  `tr` is this half-warp's 16 x 16 buffer of pairs
// (2 KB, 16-byte aligned).
__device__ __forceinline__ void rotate_pair(const uint16_t *__restrict__ blk0, const uint16_t *__restrict__ blk1,
                                            int L, uint64_t *tr, unsigned hmask, uint64_t (&v)[16])
{
    const uint4 *s0 = reinterpret_cast<const uint4 *>(blk0 + 16 * L);
    const uint4 p0 = __ldg(s0), p1 = __ldg(s0 + 1);
    uint4 q0 = make_uint4(0u, 0u, 0u, 0u), q1 = q0;
    if (blk1 != nullptr) {
        const uint4 *s1 = reinterpret_cast<const uint4 *>(blk1 + 16 * L);
        q0 = __ldg(s1);
        q1 = __ldg(s1 + 1);
    }
    const uint32_t w0[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    const uint32_t w1[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        v[2 * i] = pk(w0[i] << 16, w1[i] << 16);                      // element 2i: low bf16
        v[2 * i + 1] = pk(w0[i] & 0xFFFF0000u, w1[i] & 0xFFFF0000u);  // element 2i+1: high bf16
    }
    // stride 1 (digit d0 = b % 4), then stride 4 (digit d1 = b / 4)
#pragma unroll
    for (int q = 0; q < 4; ++q)
        h4_quad2(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
#pragma unroll
    for (int q = 0; q < 4; ++q)
        h4_quad2(v[q], v[q + 4], v[q + 8], v[q + 12]);
    // Transpose through shared memory.  Row L goes out as eight 16-byte
    // stores, pairs 2c and 2c + 1 at chunk position c ^ (L % 8); column L
    // comes back as 16 eight-byte loads.  Both sides are conflict-free.
    {
        uint4 *rowp = reinterpret_cast<uint4 *>(tr + 16 * L);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint32_t a0, a1, b0, b1;
            unpk(v[2 * c], a0, a1);
            unpk(v[2 * c + 1], b0, b1);
            rowp[c ^ (L & 7)] = make_uint4(a0, a1, b0, b1);
        }
    }
    __syncwarp(hmask);
#pragma unroll
    for (int a = 0; a < 16; ++a)
        v[a] = tr[16 * a + 2 * ((L >> 1) ^ (a & 7)) + (L & 1)];
    __syncwarp(hmask);
    // stride 16 (digit d2 = a % 4), then stride 64 (digit d3 = a / 4)
#pragma unroll
    for (int q = 0; q < 4; ++q)
        h4_quad2(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
#pragma unroll
    for (int q = 0; q < 4; ++q)
        h4_quad2(v[q], v[q + 4], v[q + 8], v[q + 12]);
    // The final 1/16 is not applied here: v holds R = 16 r.  Scaling by a power
    // of two commutes with rounding away from subnormals, so the quantiser
    // works on R with the scale multiplied by 16 and gets the same integers
    // (rows whose values reach the subnormal range take an exact path that
    // applies the 1/16 per element).
}

// max |v| over both halves of 16 pairs as a tree (fmaxf drops NaN operands, so
// the result is NaN-free and >= 0 for any inputs; max is exact in any order).
__device__ __forceinline__ float max_abs_pairs(const uint64_t (&v)[16])
{
    float m[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        uint32_t lo, hi;
        unpk(v[i], lo, hi);
        m[i] = fmaxf(fabsf(__uint_as_float(lo)), fabsf(__uint_as_float(hi)));
    }
#pragma unroll
    for (int s = 8; s >= 1; s >>= 1)
#pragma unroll
        for (int i = 0; i < s; ++i)
            m[i] = fmaxf(m[i], m[i + s]);
    return m[0];
}

// Quantise this lane's 16 column values of both blocks and store them in row
// order (dst1 == nullptr: the high halves are the zero stand-in block and are
// not stored).  v holds R = 16 r (see rotate_pair); scale is s, the row's
// scale.  `tb` is the half-warp's transpose buffer seen as bytes: block 0's
// 16 x 16 tile at +0, block 1's at +256.
//
// The arithmetic is quantise_store's, two lanes at a time, with one change to
// the near-tie test: with d = t - rint(t), an element is near a tie when
// |d| >= thr = 0.5 - 2^-15, and the packed screen tests d * d - thr^2 >= 0
// (one fused rounding, so its sign is exact; thr^2 rounded down as a float
// constant only widens the screen).  A lane whose screen fires redoes the
// elements with |d| >= thr with the exact quotient R / (16 s).
__device__ __forceinline__ void quantise_store_pair(const uint64_t (&v)[16], float scale, float inv16, int32_t qmax,
                                                    bool exact_row, int L, uint8_t *tb, unsigned hmask,
                                                    int8_t *__restrict__ dst0, int8_t *__restrict__ dst1)
{
    constexpr float kThr = 0.499969482421875f;  // 0.5 - 2^-15
    if (!exact_row) {
        const uint64_t inv2 = pk(__float_as_uint(inv16), __float_as_uint(inv16));
        const uint64_t magic2 = 0x4B4000004B400000ull;  // (1.5 * 2^23, 1.5 * 2^23)
        const uint32_t nthr = __float_as_uint(-(kThr * kThr));
        const uint64_t nthr2 = pk(nthr, nthr);
        uint32_t all_neg = 0xFFFFFFFFu;  // sign bit stays set while no element is near a tie
#pragma unroll
        for (int a = 0; a < 16; ++a) {
            const uint64_t t = mul2(v[a], inv2);
            const uint64_t tm = add2(t, magic2);
            const uint64_t d = sub2(t, sub2(tm, magic2));
            uint32_t e0, e1, b0, b1;
            unpk(fma2(d, d, nthr2), e0, e1);
            all_neg &= e0 & e1;
            unpk(tm, b0, b1);
            tb[16 * a + L] = (uint8_t)b0;
            tb[256 + 16 * a + L] = (uint8_t)b1;
        }
        if ((all_neg & 0x80000000u) == 0u) {
            const float s16 = __fmul_rn(scale, 16.0f);
#pragma unroll
            for (int a = 0; a < 16; ++a) {
                uint32_t r0, r1;
                unpk(v[a], r0, r1);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float R = __uint_as_float(h == 0 ? r0 : r1);
                    const float t = __fmul_rn(R, inv16);
                    const float d = __fsub_rn(t, __fsub_rn(__fadd_rn(t, 12582912.0f), 12582912.0f));
                    if (fabsf(d) >= kThr) {
                        const int32_t q = __float2int_rn(__fdiv_rn(R, s16));
                        tb[256 * h + 16 * a + L] = (uint8_t)min(max(q, -qmax), qmax);
                    }
                }
            }
        }
    } else {
#pragma unroll
        for (int a = 0; a < 16; ++a) {
            uint32_t r0, r1;
            unpk(v[a], r0, r1);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float r = __fmul_rn(__uint_as_float(h == 0 ? r0 : r1), 0.0625f);
                const int32_t q = __float2int_rn(__fdiv_rn(r, scale));
                tb[256 * h + 16 * a + L] = (uint8_t)min(max(q, -qmax), qmax);
            }
        }
    }
    __syncwarp(hmask);
    *reinterpret_cast<uint4 *>(dst0 + 16 * L) = *reinterpret_cast<const uint4 *>(tb + 16 * L);
    if (dst1 != nullptr)
        *reinterpret_cast<uint4 *>(dst1 + 16 * L) = *reinterpret_cast<const uint4 *>(tb + 256 + 16 * L);
    __syncwarp(hmask);
}

// Shared memory of a CTA of THREADS threads: one 2 KB transpose buffer per
// half-warp.
template <int THREADS>
constexpr int smem_bytes()
{
    return (THREADS / 16) * 256 * 8;
}

// THREADS / 16 half-warps per row, each holding up to J block pairs in
// registers (kRecompute: one at a time, rotating every pair twice).
template <int J, bool kRecompute, int THREADS>
__global__ void __launch_bounds__(THREADS) rotquant_pairs_kernel(const uint16_t *__restrict__ x, int64_t M,
                                                                  int64_t K, int qmax, int8_t *__restrict__ xq,
                                                                  float *__restrict__ xs)
{
    constexpr int kHalfWarps = THREADS / 16;  // block pairs in flight per CTA
    extern __shared__ __align__(16) uint64_t rq_smem[];
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
    const int NP = (NB + 1) / 2;  // block pairs (2p, 2p + 1); the last one may be alone
    int8_t *__restrict__ qrow = xq + m * K;

    if (m >= M) {  // padding row of the decode GEMV operand
        for (int64_t c = tid; c < K / 16; c += THREADS)
            reinterpret_cast<uint4 *>(qrow)[c] = make_uint4(0u, 0u, 0u, 0u);
        if (tid == 0)
            xs[m] = 1.0f;
        return;
    }

    const uint16_t *__restrict__ xrow = x + m * K;
    uint64_t *tr = rq_smem + 256 * hw;
    // the same buffer serves the byte transpose; the odd half-warp's byte
    // tiles start 64 bytes in, so that the byte stores of a warp's two
    // half-warps fall in different banks
    uint8_t *tb = reinterpret_cast<uint8_t *>(tr) + 64 * (hw & 1);
    float amax = 0.0f;
    uint64_t v[kRecompute ? 1 : J][16];
    // the second block of pair p, or nullptr where the row ends with a lone block
    auto src1 = [&](int p) { return 2 * p + 1 < NB ? xrow + 256 * (2 * p + 1) : nullptr; };
    auto dst1 = [&](int p) { return 2 * p + 1 < NB ? qrow + 256 * (2 * p + 1) : nullptr; };

    if (!kRecompute) {
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int p = hw + kHalfWarps * j;
            if (p < NP) {
                rotate_pair(xrow + 512 * p, src1(p), L, tr, hmask, v[j]);
                amax = fmaxf(amax, max_abs_pairs(v[j]));
            }
        }
    } else {
        for (int p = hw; p < NP; p += kHalfWarps) {
            rotate_pair(xrow + 512 * p, src1(p), L, tr, hmask, v[0]);
            amax = fmaxf(amax, max_abs_pairs(v[0]));
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
            const int p = hw + kHalfWarps * j;
            if (p < NP)
                quantise_store_pair(v[j], scale, inv16, qmax, exact_row, L, tb, hmask, qrow + 512 * p, dst1(p));
        }
    } else {
        for (int p = hw; p < NP; p += kHalfWarps) {
            rotate_pair(xrow + 512 * p, src1(p), L, tr, hmask, v[0]);
            quantise_store_pair(v[0], scale, inv16, qmax, exact_row, L, tb, hmask, qrow + 512 * p, dst1(p));
        }
    }
    if (tid == 0)
        xs[m] = scale;
}

using KernelFn = void (*)(const uint16_t *, int64_t, int64_t, int, int8_t *, float *);

// Opt the kernels whose dynamic shared memory passes 48 KB into the larger
// size: the packed form's 384- and 512-thread CTAs (transpose buffers) and
// every short-batch kernel (its reservation).  Once per device, before the
// first launch.
inline cudaError_t set_attributes()
{
    struct Need {
        KernelFn f;
        int bytes;
    };
    const Need need[] = {
        {rotquant_pairs_kernel<1, false, 512>, smem_bytes<512>()},
        {rotquant_pairs_kernel<2, false, 512>, smem_bytes<512>()},
        {rotquant_pairs_kernel<1, true, 512>, smem_bytes<512>()},
        {rotquant_pairs_kernel<1, false, 384>, smem_bytes<384>()},
        {rotquant_rows_kernel<1, false, 256>, kShortReserve},
        {rotquant_rows_kernel<2, false, 256>, kShortReserve},
        {rotquant_rows_kernel<3, false, 256>, kShortReserve},
        {rotquant_rows_kernel<4, false, 256>, kShortReserve},
        {rotquant_rows_kernel<1, true, 256>, kShortReserve},
        {rotquant_rows_kernel<1, false, 512>, kShortReserve},
        {rotquant_rows_kernel<2, false, 512>, kShortReserve},
        {rotquant_rows_kernel<3, false, 512>, kShortReserve},
        {rotquant_rows_kernel<4, false, 512>, kShortReserve},
        {rotquant_rows_kernel<1, true, 512>, kShortReserve},
    };
    for (const Need &n : need) {
        const cudaError_t e = cudaFuncSetAttribute(n.f, cudaFuncAttributeMaxDynamicSharedMemorySize, n.bytes);
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

template <int J, bool kRecompute, int THREADS>
inline cudaError_t launch_t(const uint16_t *x, int64_t M, int64_t K, int64_t MP, int qmax, int8_t *xq, float *xs,
                            cudaStream_t stream)
{
    // a programmatic dependent of the previous kernel on the stream: its
    // launch overlaps that kernel's tail, and the kernel waits for it
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)MP);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem_bytes<THREADS>();
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, rotquant_pairs_kernel<J, kRecompute, THREADS>, x, M, K, qmax, xq, xs);
}

// One CTA per row.  Short batches: the scalar form, 512 threads for K >= 8192
// and 256 below.  Otherwise the packed form with one half-warp per block pair
// where that fits in 512 threads (K <= 16384; the CTA size follows the row:
// 64 to 512 threads), two pairs per half-warp up to K = 32768, and the
// recomputing second pass beyond.
inline cudaError_t launch(const uint16_t *x, int64_t M, int64_t K, int64_t MP, int qmax, int8_t *xq, float *xs,
                          cudaStream_t stream)
{
    if (MP <= kShortRows)
        return K >= 8192 ? launch_rows_t<512>(x, M, K, MP, qmax, xq, xs, stream)
                         : launch_rows_t<256>(x, M, K, MP, qmax, xq, xs, stream);
    const int64_t pairs = (K / 256 + 1) / 2;
    if (pairs <= 4)
        return launch_t<1, false, 64>(x, M, K, MP, qmax, xq, xs, stream);
    if (pairs <= 8)
        return launch_t<1, false, 128>(x, M, K, MP, qmax, xq, xs, stream);
    if (pairs <= 16)
        return launch_t<1, false, 256>(x, M, K, MP, qmax, xq, xs, stream);
    if (pairs <= 24)
        return launch_t<1, false, 384>(x, M, K, MP, qmax, xq, xs, stream);
    if (pairs <= 32)
        return launch_t<1, false, 512>(x, M, K, MP, qmax, xq, xs, stream);
    if (pairs <= 64)
        return launch_t<2, false, 512>(x, M, K, MP, qmax, xq, xs, stream);
    return launch_t<1, true, 512>(x, M, K, MP, qmax, xq, xs, stream);
}

}  // namespace rq
}  // namespace cr
