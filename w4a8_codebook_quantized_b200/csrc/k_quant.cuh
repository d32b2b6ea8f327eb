// Offline quantiser of the W4A8 codebook layer: rotated fp32 weights ->
// packed 4-bit codes, fp8 e4m3fn group scales and per-channel scales.
//
// ai-toolkit convrot_w4a8_quant.py, quantize_w4a8_rotated /
// _quantize_rotated_rows (group absmax, nearest codebook index, _ALS_ITERS =
// 2 least-squares refinements of the group scale, s_channel from the row's
// largest |codebook[code] * gs| / 127, s_rel = fp8(gs / s_channel), final
// codes = nearest level of w / s_channel on grid_levels(s_rel)), and
// requantize_codes_ without its rotation (_assign_grid, deterministic or
// stochastic, on stored scales).
//
// Every decision is a floating-point comparison, so each value is computed
// with the same IEEE operations in the same order as the plain definition:
// divisions are __fdiv_rn, products and sums __fmul_rn / __fadd_rn (never
// contracted), the group sums of 16 products pairwise ((p0 + p1) + (p2 + p3))
// and so on up.  "Nearest" is the pages' search + neighbour rule: pos = the
// number of levels strictly below x (the levels are sorted), lo = pos - 1 and
// hi = pos clamped to the table, the fp32 distances |x - level|, and the upper
// level only when strictly nearer.
#pragma once

#include <cstdint>

#include "cr_device.cuh"

namespace cr {
namespace qz {

constexpr int kThreads = 256;
constexpr int kLvStride = 17;  // floats per thread in the level table (odd: no bank conflicts)
constexpr float kEps = 1e-8f;  // the pages' clamp(min=1e-8), as an fp32

__device__ __forceinline__ float clamp_min(float v, float lo)
{
    return v < lo ? lo : v;  // NaN stays NaN, as torch's clamp
}

// Number of the 16 sorted values of `t` (shared memory, stride 1) strictly
// below x: a branchless lower bound in four halving steps and one last test.
__device__ __forceinline__ int count_below16(const float *t, float x)
{
    int pos = 0;
#pragma unroll
    for (int s = 8; s >= 1; s >>= 1)
        pos += (t[pos + s - 1] < x) ? s : 0;
    if (pos == 15 && t[15] < x)
        pos = 16;
    return pos;
}

// The nearest of the 16 sorted values of `t` to x (ties to the lower).
__device__ __forceinline__ int nearest16(const float *t, float x)
{
    const int pos = count_below16(t, x);
    const int lo = pos - 1 < 0 ? 0 : (pos - 1 > 15 ? 15 : pos - 1);
    const int hi = pos > 15 ? 15 : pos;
    const float dlo = fabsf(__fsub_rn(x, t[lo]));
    const float dhi = fabsf(__fsub_rn(x, t[hi]));
    return dhi < dlo ? hi : lo;
}

// The stochastic choice between the two levels bracketing x, with the uniform
// draw u: threshold u * width + level_lo (two roundings), upper when x is
// strictly above it.
__device__ __forceinline__ int stochastic16(const float *t, float x, float u)
{
    const int pos = count_below16(t, x);
    int lo = pos - 1;
    lo = lo < 0 ? 0 : (lo > 14 ? 14 : lo);
    const float level_lo = t[lo];
    const float width = __fsub_rn(t[lo + 1], level_lo);
    const float thr = __fadd_rn(__fmul_rn(u, width), level_lo);
    const int code = lo + (x > thr ? 1 : 0);
    return code > 15 ? 15 : code;
}

// fp32 -> fp8 e4m3fn with torch's conversion semantics: nearest e4m3 value,
// ties to even; a magnitude that rounds to 480 or more (the NaN pattern
// S.1111.111), an infinity or a NaN gives NaN (0x7F | sign); no saturation.
// Below 2^-6 the value is a multiple of 2^-9 (subnormals), rounded the same
// way.
__device__ __forceinline__ uint8_t f32_to_fp8_e4m3fn(float f)
{
    uint32_t bits = __float_as_uint(f);
    const uint32_t sign = (bits >> 24) & 0x80u;
    bits &= 0x7FFFFFFFu;
    if (bits >= 0x43F00000u)  // >= 480.0, +inf or NaN
        return (uint8_t)(sign | 0x7Fu);
    if (bits < 0x3C800000u) {  // below 2^-6: units of 2^-9, exact scaling
        const int r = __float2int_rn(__fmul_rn(__uint_as_float(bits), 512.0f));
        return (uint8_t)(sign | (uint32_t)r);
    }
    // keep 3 mantissa bits, round to nearest even, rebias 127 -> 7
    const uint32_t odd = (bits >> 20) & 1u;
    const uint32_t r = (bits + 0x7FFFFu + odd) >> 20;
    return (uint8_t)(sign | (r - (120u << 3)));
}

__device__ __forceinline__ float fp8_e4m3fn_to_f32(uint8_t b)
{
    const uint32_t sign = (uint32_t)(b & 0x80u) << 24;
    const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
    if (e == 0xFu && m == 7u)
        return __uint_as_float(sign | 0x7FC00000u);
    if (e == 0u) {  // m * 2^-9 (exact)
        const float v = __fmul_rn((float)m, 1.0f / 512.0f);
        return sign ? -v : v;
    }
    return __uint_as_float(sign | ((e + 120u) << 23) | (m << 20));
}

// grid_levels of one fp8 scale byte into t[0..15]: clamp(rint(cb[i] * s), +-127).
__device__ __forceinline__ void grid_levels16(const float *cb, uint8_t srel, float *t)
{
    const float s = fp8_e4m3fn_to_f32(srel);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float v = rintf(__fmul_rn(cb[i], s));
        v = v < -127.0f ? -127.0f : v;
        v = v > 127.0f ? 127.0f : v;
        t[i] = v;
    }
}

__device__ __forceinline__ float sum16_pairwise(const float (&v)[16])
{
    float a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        a[i] = __fadd_rn(v[2 * i], v[2 * i + 1]);
    const float b0 = __fadd_rn(a[0], a[1]), b1 = __fadd_rn(a[2], a[3]);
    const float b2 = __fadd_rn(a[4], a[5]), b3 = __fadd_rn(a[6], a[7]);
    return __fadd_rn(__fadd_rn(b0, b1), __fadd_rn(b2, b3));
}

__device__ __forceinline__ void load16(const float *__restrict__ p, float (&w)[16])
{
    const float4 *p4 = reinterpret_cast<const float4 *>(p);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float4 v = p4[j];
        w[4 * j] = v.x;
        w[4 * j + 1] = v.y;
        w[4 * j + 2] = v.z;
        w[4 * j + 3] = v.w;
    }
}

// One CTA per row (grid-stride): phase A computes every group's scale after
// the ALS passes (kept in shared memory) and the row maximum of
// |codebook[code] * gs|; phase B writes s_channel, each group's fp8 scale and
// its 16 final codes, packed two to a byte (column 2j in the low nibble).
// Dynamic shared memory: G = K / 16 floats of group scales.
__global__ void __launch_bounds__(kThreads) quantize_kernel(const float *__restrict__ w_rot,
                                                            const float *__restrict__ codebook, int64_t N, int K,
                                                            uint8_t *__restrict__ qdata, uint8_t *__restrict__ srel,
                                                            float *__restrict__ s_channel)
{
    extern __shared__ float gs_s[];
    __shared__ float cb[16];
    __shared__ float lv_s[kThreads * kLvStride];
    __shared__ float red[kThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = K >> 4;
    if (tid < 16)
        cb[tid] = codebook[tid];
    __syncthreads();
    float *lv = lv_s + tid * kLvStride;

    for (int64_t n = blockIdx.x; n < N; n += gridDim.x) {
        const float *row = w_rot + n * (int64_t)K;
        float rmax = 0.0f;
        for (int g = tid; g < G; g += kThreads) {
            float w[16];
            load16(row + 16 * g, w);
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i)
                amax = fabsf(w[i]) > amax ? fabsf(w[i]) : amax;
            float gs = clamp_min(amax, kEps);
            int q[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                q[i] = nearest16(cb, __fdiv_rn(w[i], gs));
#pragma unroll 1
            for (int it = 0; it < 2; ++it) {
                float p[16], l2[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float l = cb[q[i]];
                    p[i] = __fmul_rn(w[i], l);
                    l2[i] = __fmul_rn(l, l);
                }
                const float num = sum16_pairwise(p);
                const float den = clamp_min(sum16_pairwise(l2), kEps);
                gs = clamp_min(__fdiv_rn(num, den), kEps);
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    q[i] = nearest16(cb, __fdiv_rn(w[i], gs));
            }
            gs_s[g] = gs;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float a = fabsf(__fmul_rn(cb[q[i]], gs));
                rmax = a > rmax ? a : rmax;
            }
        }
        // row maximum (a maximum is exact in any order)
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float v = __shfl_xor_sync(0xffffffffu, rmax, o);
            rmax = v > rmax ? v : rmax;
        }
        if (lane == 0)
            red[warp] = rmax;
        __syncthreads();
        float m = red[0];
#pragma unroll
        for (int i = 1; i < kThreads / 32; ++i)
            m = red[i] > m ? red[i] : m;
        const float sch = clamp_min(__fdiv_rn(m, 127.0f), kEps);
        if (tid == 0)
            s_channel[n] = sch;

        for (int g = tid; g < G; g += kThreads) {
            const uint8_t sb = f32_to_fp8_e4m3fn(__fdiv_rn(gs_s[g], sch));
            srel[n * (int64_t)G + g] = sb;
            grid_levels16(cb, sb, lv);
            float w[16];
            load16(row + 16 * g, w);
            uint32_t packed[2] = {0u, 0u};
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t c = (uint32_t)nearest16(lv, __fdiv_rn(w[i], sch));
                packed[i >> 3] |= c << (4 * (i & 7));
            }
            *reinterpret_cast<uint2 *>(qdata + n * (int64_t)(K / 2) + 8 * g) = make_uint2(packed[0], packed[1]);
        }
        __syncthreads();  // red and gs_s are reused by the next row
    }
}

// Codes on stored scales, one thread per group of 16 (grid-stride):
// target = w_rot / s_channel, levels = grid_levels(s_rel); nearest level, or
// the stochastic choice with rand[n, k] when rand is given.
__global__ void __launch_bounds__(kThreads) assign_kernel(const float *__restrict__ w_rot,
                                                          const uint8_t *__restrict__ srel,
                                                          const float *__restrict__ s_channel,
                                                          const float *__restrict__ codebook,
                                                          const float *__restrict__ rand, int64_t N, int K,
                                                          uint8_t *__restrict__ qdata)
{
    __shared__ float cb[16];
    __shared__ float lv_s[kThreads * kLvStride];
    const int tid = threadIdx.x;
    if (tid < 16)
        cb[tid] = codebook[tid];
    __syncthreads();
    float *lv = lv_s + tid * kLvStride;
    const int G = K >> 4;
    const int64_t total = N * (int64_t)G;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + tid; i < total; i += (int64_t)gridDim.x * kThreads) {
        const int64_t n = i / G;
        const int g = (int)(i - n * G);
        grid_levels16(cb, srel[i], lv);
        const float sch = s_channel[n];
        const int64_t base = n * (int64_t)K + 16 * g;
        float w[16];
        load16(w_rot + base, w);
        float u[16];
        if (rand != nullptr)
            load16(rand + base, u);
        uint32_t packed[2] = {0u, 0u};
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float t = __fdiv_rn(w[j], sch);
            const uint32_t c = (uint32_t)(rand != nullptr ? stochastic16(lv, t, u[j]) : nearest16(lv, t));
            packed[j >> 3] |= c << (4 * (j & 7));
        }
        *reinterpret_cast<uint2 *>(qdata + n * (int64_t)(K / 2) + 8 * g) = make_uint2(packed[0], packed[1]);
    }
}

inline size_t quantize_smem_bytes(int K)
{
    return (size_t)(K / 16) * sizeof(float);
}

inline cudaError_t launch_quantize(const float *w_rot, const float *codebook, int64_t N, int K, uint8_t *qdata,
                                   uint8_t *srel, float *s_channel, int num_sms, cudaStream_t stream)
{
    const size_t smem = quantize_smem_bytes(K);
    cudaError_t e = cudaFuncSetAttribute(quantize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    const int64_t cap = (int64_t)num_sms * 4;
    const int grid = (int)(N < cap ? N : cap);
    quantize_kernel<<<grid, kThreads, smem, stream>>>(w_rot, codebook, N, K, qdata, srel, s_channel);
    return cudaGetLastError();
}

inline cudaError_t launch_assign(const float *w_rot, const uint8_t *srel, const float *s_channel,
                                 const float *codebook, const float *rand, int64_t N, int K, uint8_t *qdata,
                                 int num_sms, cudaStream_t stream)
{
    const int64_t groups = N * (int64_t)(K / 16);
    int64_t blocks = (groups + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)num_sms * 4;
    blocks = blocks < cap ? blocks : cap;
    blocks = blocks < 1 ? 1 : blocks;
    assign_kernel<<<(unsigned)blocks, kThreads, 0, stream>>>(w_rot, srel, s_channel, codebook, rand, N, K, qdata);
    return cudaGetLastError();
}

}  // namespace qz
}  // namespace cr
