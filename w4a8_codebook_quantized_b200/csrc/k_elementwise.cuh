// k_elementwise.cuh -- the two bandwidth-bound stand-alone kernels: decode of
// the packed codes onto the int8 grid, and the epilogue on an int32
// accumulator.
#pragma once

#include "cr_device.cuh"

namespace cr {
namespace ew {

constexpr int kThreads = 256;

// ai-toolkit convrot_w4a8_quant.py, unpack_w4a8_eager / w4a8_unpack_kernel:
// w8[n, k] = sat_s8(rne(codebook[code] * fp8(srel[n, k/16]))).
//
// Grid-stride over groups: a thread takes one group of 16 weights (8 bytes
// of codes, one scale byte) and writes its 16 output bytes, so a warp's store
// is one contiguous 512-byte run of whole sectors (two 16-byte stores per
// 32-byte chunk, one per half-sector, were written back to DRAM about 2.6
// times over).  Each thread issues the loads of kDecodeUnroll groups before it
// decodes any, to keep enough bytes in flight; per group one lookup in the
// CTA's level table (4 copies, the copy chosen by lane, to spread a
// quarter-warp's lookups over bank groups) and two byte-permute decodes.
// HBM traffic per weight: 0.5 + 1/16 bytes in, 1 byte out.
constexpr int kDecodeUnroll = 8;
constexpr int kDecodeLutCopies = 4;

__global__ void __launch_bounds__(kThreads) decode_int8_kernel(const uint8_t *__restrict__ qdata,
                                                               const uint8_t *__restrict__ srel,
                                                               const float *__restrict__ codebook, int64_t N,
                                                               int64_t K, int8_t *__restrict__ w8)
{
    __shared__ uint4 lut[256 * kDecodeLutCopies];
    __shared__ float cb[16];
    if (threadIdx.x < 16)
        cb[threadIdx.x] = codebook[threadIdx.x];
    __syncthreads();
    for (int s = threadIdx.x; s < 256; s += kThreads) {
        const uint4 e = lut_entry((uint32_t)s, cb);
#pragma unroll
        for (int c = 0; c < kDecodeLutCopies; ++c)
            lut[s * kDecodeLutCopies + c] = e;
    }
    __syncthreads();

    const uint4 *lutc = lut + (threadIdx.x & (kDecodeLutCopies - 1));
    // groups are contiguous across rows: group i has its codes at 8 i, its
    // scale byte at i and its output at 16 i
    const int64_t total = N * (K / 16);
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t i0 = (int64_t)blockIdx.x * kThreads + threadIdx.x; i0 < total; i0 += kDecodeUnroll * stride) {
        uint2 c[kDecodeUnroll];
        uint32_t sb[kDecodeUnroll];
#pragma unroll
        for (int u = 0; u < kDecodeUnroll; ++u) {
            const int64_t i = i0 + u * stride;
            if (i < total) {
                c[u] = ldg_stream8(qdata + 8 * i);
                sb[u] = __ldg(srel + i);
            }
        }
#pragma unroll
        for (int u = 0; u < kDecodeUnroll; ++u) {
            const int64_t i = i0 + u * stride;
            if (i < total) {
                const uint4 T = lutc[kDecodeLutCopies * sb[u]];
                uint4 o;
                decode8(c[u].x, T, o.x, o.y);
                decode8(c[u].y, T, o.z, o.w);
                *reinterpret_cast<uint4 *>(w8 + 16 * i) = o;
            }
        }
    }
}

inline cudaError_t launch_decode(const uint8_t *qdata, const uint8_t *srel, const float *codebook, int64_t N,
                                 int64_t K, int8_t *w8, int num_sms, cudaStream_t stream)
{
    const int64_t total = N * (K / 16);
    int64_t blocks = (total + (int64_t)kThreads * kDecodeUnroll - 1) / ((int64_t)kThreads * kDecodeUnroll);
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap)
        blocks = cap;
    decode_int8_kernel<<<(unsigned)blocks, kThreads, 0, stream>>>(qdata, srel, codebook, N, K, w8);
    return cudaGetLastError();
}

// ai-toolkit convrot_w4a8_quant.py, w4a8_gemv_kernel epilogue, on a stored
// int32 accumulator.  Four outputs per thread along a row when N % 4 == 0
// (16-byte accumulator loads), one otherwise.
__global__ void __launch_bounds__(kThreads) epilogue_kernel(const int32_t *__restrict__ acc,
                                                            const float *__restrict__ xs,
                                                            const float *__restrict__ ws,
                                                            const float *__restrict__ bias, int64_t M, int64_t N,
                                                            int out_f32, void *__restrict__ out)
{
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    if ((N & 3) == 0) {
        const int64_t total = M * N / 4;
        for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < total; i += stride) {
            const int64_t e = 4 * i;
            const int64_t m = e / N, n = e - m * N;
            const int4 a = __ldg(reinterpret_cast<const int4 *>(acc) + i);
            const float xm = xs[m];
            const float y0 = epilogue_value(a.x, xm, ws[n], bias, n);
            const float y1 = epilogue_value(a.y, xm, ws[n + 1], bias, n + 1);
            const float y2 = epilogue_value(a.z, xm, ws[n + 2], bias, n + 2);
            const float y3 = epilogue_value(a.w, xm, ws[n + 3], bias, n + 3);
            if (out_f32) {
                reinterpret_cast<float4 *>(out)[i] = make_float4(y0, y1, y2, y3);
            } else {
                const uint32_t lo = (uint32_t)to_bf16_bits(y0) | ((uint32_t)to_bf16_bits(y1) << 16);
                const uint32_t hi = (uint32_t)to_bf16_bits(y2) | ((uint32_t)to_bf16_bits(y3) << 16);
                reinterpret_cast<uint2 *>(out)[i] = make_uint2(lo, hi);
            }
        }
    } else {
        const int64_t total = M * N;
        for (int64_t e = (int64_t)blockIdx.x * kThreads + threadIdx.x; e < total; e += stride) {
            const int64_t m = e / N, n = e - m * N;
            const float y = epilogue_value(acc[e], xs[m], ws[n], bias, n);
            if (out_f32)
                reinterpret_cast<float *>(out)[e] = y;
            else
                reinterpret_cast<uint16_t *>(out)[e] = to_bf16_bits(y);
        }
    }
}

inline cudaError_t launch_epilogue(const int32_t *acc, const float *xs, const float *ws, const float *bias,
                                   int64_t M, int64_t N, int out_f32, void *out, int num_sms, cudaStream_t stream)
{
    const int64_t work = ((N & 3) == 0) ? M * N / 4 : M * N;
    int64_t blocks = (work + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap)
        blocks = cap;
    if (blocks < 1)
        blocks = 1;
    epilogue_kernel<<<(unsigned)blocks, kThreads, 0, stream>>>(acc, xs, ws, bias, M, N, out_f32, out);
    return cudaGetLastError();
}

// ---------------------------------------------------------------- row interleave
//
// h3-rs weights.rs, interleave_rows: the two halves of the row dimension,
// rows [0, F) and [F, 2F), become pairs: dst row 2f = src row f and dst row
// 2f + 1 = src row F + f.  Applied to a gate/up layer's qdata, srel,
// s_channel and bias it gives the row order the SwiGLU epilogues read.  A
// grid-stride copy in units of V bytes (16, 4 or 1, the largest that divides
// the row and both addresses).
template <class V>
__global__ void __launch_bounds__(kThreads) interleave_rows_kernel(const V *__restrict__ src, V *__restrict__ dst,
                                                                   int64_t rows, int64_t units_per_row)
{
    const int64_t half = rows >> 1, total = rows * units_per_row;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t drow = i / units_per_row, c = i - drow * units_per_row;
        const int64_t srow = (drow & 1) ? half + (drow >> 1) : (drow >> 1);
        dst[i] = src[srow * units_per_row + c];
    }
}

inline cudaError_t launch_interleave_rows(const void *src, void *dst, int64_t rows, int64_t row_bytes, int num_sms,
                                          cudaStream_t stream)
{
    const uintptr_t align = (uintptr_t)src | (uintptr_t)dst | (uintptr_t)row_bytes;
    const int vec = (align & 15) == 0 ? 16 : (align & 3) == 0 ? 4 : 1;
    const int64_t units = row_bytes / vec, total = rows * units;
    int64_t blocks = (total + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap)
        blocks = cap;
    if (blocks < 1)
        blocks = 1;
    if (vec == 16)
        interleave_rows_kernel<uint4><<<(unsigned)blocks, kThreads, 0, stream>>>(
            static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), rows, units);
    else if (vec == 4)
        interleave_rows_kernel<uint32_t><<<(unsigned)blocks, kThreads, 0, stream>>>(
            static_cast<const uint32_t *>(src), static_cast<uint32_t *>(dst), rows, units);
    else
        interleave_rows_kernel<uint8_t><<<(unsigned)blocks, kThreads, 0, stream>>>(
            static_cast<const uint8_t *>(src), static_cast<uint8_t *>(dst), rows, units);
    return cudaGetLastError();
}

// ---------------------------------------------------------------- backward weight
//
// ai-toolkit convrot_w4a8_quant.py, _w4a8_linear_ste_backward: the weight of
// the input gradient, w = w8.to(bf16) * s_channel.to(bf16), here written
// transposed, wt[k, n] = bf16(w8[n, k] * bf16(s_channel[n])) [K, N], the
// K-major B operand of dx = grad @ w.  w8 is the forward's decode (the same
// per-CTA table of 16 int8 levels per scale byte and byte permutes); the
// product of an int8 and a bf16 is exact in fp32 and is rounded once.
// A CTA per 64 (n) x 128 (k) tile: thread (g = tid / 32, p = tid % 32)
// decodes group g (16 columns) of rows n0 + 2p and n0 + 2p + 1 and stores
// the 16 bf16 pairs (row 2p, row 2p + 1) of those columns into a shared tile
// of 4-byte pairs [128 k][36] (lanes on consecutive pairs: no bank
// conflicts); the tile then leaves as 128 rows of 64 bf16 (16-byte stores, 8
// lanes per 128-byte row).  N must be a multiple of 8 and K of 128.
constexpr int kTN = 64, kTK = 128, kTPairs = 36;  // 32 row pairs + 4 of padding (16-byte aligned rows)

__global__ void __launch_bounds__(kThreads) dequant_t_bf16_kernel(const uint8_t *__restrict__ qdata,
                                                                  const uint8_t *__restrict__ srel,
                                                                  const float *__restrict__ codebook,
                                                                  const float *__restrict__ s_channel, int N, int K,
                                                                  uint16_t *__restrict__ wt)
{
    __shared__ __align__(16) uint32_t tile[kTK][kTPairs];
    __shared__ uint4 lut[256];
    __shared__ float cb[16];
    if (threadIdx.x < 16)
        cb[threadIdx.x] = codebook[threadIdx.x];
    __syncthreads();
    lut[threadIdx.x] = lut_entry(threadIdx.x, cb);  // kThreads == 256 scale bytes
    __syncthreads();
    const int tiles_k = K / kTK, tiles_n = (N + kTN - 1) / kTN;
    const int p = threadIdx.x & 31, g = threadIdx.x >> 5;
    // n fastest: CTAs running together write neighbouring 128-byte strips of
    // the same 128 rows of wt (whole rows between them), not one strip each
    // of rows 8 KB apart
    for (int t = blockIdx.x; t < tiles_k * tiles_n; t += gridDim.x) {
        const int tk = t / tiles_n, tn = t - tk * tiles_n;
        const int n0 = tn * kTN, k0 = tk * kTK, n = n0 + 2 * p;
        if (n < N) {  // N % 8 == 0: both rows of the pair exist
            const int kg = k0 / 16 + g;  // this thread's group
            uint32_t lo[4], hi[4];
            float sch[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const uint2 c = *reinterpret_cast<const uint2 *>(qdata + (int64_t)(n + r) * (K / 2) + 8 * kg);
                const uint4 T = lut[srel[(int64_t)(n + r) * (K / 16) + kg]];
                uint32_t *w = r ? hi : lo;
                decode8(c.x, T, w[0], w[1]);
                decode8(c.y, T, w[2], w[3]);
                sch[r] = __bfloat162float(__float2bfloat16_rn(s_channel[n + r]));
            }
            // int8 -> fp32 without the conversion unit: with the sign bit
            // flipped, byte j is w + 128 in 0..255; placed as the low mantissa
            // byte of 2^23 (bits 0x4B000000) it reads as 2^23 + w + 128, and
            // subtracting 2^23 + 128 leaves w exactly
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const uint32_t sel = 0x7650u | (uint32_t)(j & 3);
                const uint32_t ab = prmt(lo[j >> 2] ^ 0x80808080u, 0x4B000000u, sel);
                const uint32_t bb = prmt(hi[j >> 2] ^ 0x80808080u, 0x4B000000u, sel);
                const float a = __fsub_rn(__uint_as_float(ab), 8388736.0f);
                const float b = __fsub_rn(__uint_as_float(bb), 8388736.0f);
                const __nv_bfloat162 v = __floats2bfloat162_rn(__fmul_rn(a, sch[0]), __fmul_rn(b, sch[1]));
                tile[16 * g + j][p] = *reinterpret_cast<const uint32_t *>(&v);
            }
        }
        __syncthreads();
        for (int i = threadIdx.x; i < kTK * (kTN / 8); i += kThreads) {
            const int kr = i >> 3, ch = i & 7, nn = n0 + 8 * ch;
            if (nn < N)  // N % 8 == 0: a 16-byte chunk is wholly inside or outside
                *reinterpret_cast<uint4 *>(wt + (int64_t)(k0 + kr) * N + nn) =
                    *reinterpret_cast<const uint4 *>(&tile[kr][4 * ch]);
        }
        __syncthreads();
    }
}

inline cudaError_t launch_dequant_t_bf16(const uint8_t *qdata, const uint8_t *srel, const float *codebook,
                                         const float *s_channel, int N, int K, uint16_t *wt, int num_sms,
                                         cudaStream_t stream)
{
    const int64_t tiles = (int64_t)(K / kTK) * ((N + kTN - 1) / kTN);
    const int64_t cap = (int64_t)num_sms * 8;
    const int grid = (int)(tiles < cap ? tiles : cap);
    dequant_t_bf16_kernel<<<grid < 1 ? 1 : grid, kThreads, 0, stream>>>(qdata, srel, codebook, s_channel, N, K, wt);
    return cudaGetLastError();
}

// ---------------------------------------------------------------- failure-path self-test
//
// Copy between page-locked host memory that the device can address and
// device memory, done by the SMs with 16-byte accesses: one vector per thread
// per pass, the grid spread wide so that no SM holds many host-link requests
// in flight.  For the tens of kilobytes of a decode step's activations and
// outputs this takes a fraction of the time of a copy-engine transfer queued
// between kernels on the same stream.  Host addresses are read with
// ld.global.cv (fetched again, never a stale cached line) and written with
// st.global.wt (write-through to system memory).
//
// Launched as a programmatic dependent of the previous kernel on the stream.
// Host to device: the host loads are issued before waiting for that kernel
// (the host wrote the source before queuing the call) and the device stores
// after it.  Device to host: the loads wait for that kernel, which produced
// the source.
constexpr int kCopyThreads = 128;

template <bool kToDevice>
__global__ void __launch_bounds__(kCopyThreads) host_copy_kernel(uint4 *__restrict__ dst,
                                                                 const uint4 *__restrict__ src, int64_t n16)
{
    asm volatile("griddepcontrol.launch_dependents;" :::);
    const int64_t stride = (int64_t)gridDim.x * kCopyThreads;
    const int64_t i0 = (int64_t)blockIdx.x * kCopyThreads + threadIdx.x;
    if (kToDevice) {
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (i0 < n16)
            v = __ldcv(src + i0);
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (i0 < n16)
            dst[i0] = v;
        for (int64_t i = i0 + stride; i < n16; i += stride)
            dst[i] = __ldcv(src + i);
    } else {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        for (int64_t i = i0; i < n16; i += stride)
            __stwt(dst + i, src[i]);
    }
}

inline cudaError_t launch_host_copy(void *dst, const void *src, int64_t bytes, bool to_device, int num_sms,
                                    cudaStream_t stream)
{
    const int64_t n16 = bytes / 16;
    const int64_t want = (n16 + kCopyThreads - 1) / kCopyThreads;
    const int64_t cap = 4 * (int64_t)num_sms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(want < cap ? want : cap));
    cfg.blockDim = dim3(kCopyThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (to_device)
        return cudaLaunchKernelEx(&cfg, host_copy_kernel<true>, reinterpret_cast<uint4 *>(dst),
                                  reinterpret_cast<const uint4 *>(src), n16);
    return cudaLaunchKernelEx(&cfg, host_copy_kernel<false>, reinterpret_cast<uint4 *>(dst),
                              reinterpret_cast<const uint4 *>(src), n16);
}

// A wait that nothing completes: one thread initialises an mbarrier expecting
// one arrival that never comes and waits for its first phase with the
// library's bounded wait.  The wait runs out after limit_ns, sets the device
// error word (as any of the pipelines' waits would) and the kernel returns:
// the error path is exercised without a fault, a trap or a hang.
__global__ void selftest_timeout_kernel(uint64_t limit_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        volatile int *ab = &abort_flag;
        mbar_wait_bounded(&bar, 0u, ab, limit_ns);
    }
}

}  // namespace ew
}  // namespace cr
