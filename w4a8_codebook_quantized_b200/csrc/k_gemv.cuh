// k_gemv.cuh -- fused decode GEMV for M <= 8 tokens.
//
// What it computes (ai-toolkit convrot_w4a8_quant.py, w4a8_gemv_kernel):
// out[m, n] = epilogue(sum_k xq[m, k] * w8[n, k]) with w8 decoded on the fly
// from the packed codes, the fp8 group scales and the codebook, so the weight
// costs 4.5 bits of HBM traffic and is never materialised.  The int32 sums
// are exact, so the result equals the prefill path bit for bit.
//
// B200 design.  The page's kernel multiply-accumulates with int32 IMAD in
// registers.  Here the decoded int8 weights stay in registers too, but the
// dot products go to the warp-level int8 tensor-core instruction
// (mma.sync m16n8k32, A = 16 weight rows x 32 k, B = 32 k x 8 tokens), fed
// directly from registers: no shared-memory round trip, and the ALU budget
// per weight drops to the decode itself (about 1.4 instructions), which
// keeps the kernel memory-bound at M = 8.  (The tcgen05 path would need the
// operands in shared memory; at 8 tokens the tensor work is negligible.)
//
// Since the sum runs over k, any permutation of k is allowed as long as A and
// B use the same one.  Thread (g = lane / 4, t = lane % 4) loads 16 contiguous
// bytes (32 codes) of weight rows g and g + 8 for k in [128 s + 32 t, +32) of
// slice s, and the matching 32 activation bytes of token g; code word i
// (columns 8i..8i+7) feeds MMA i: its first four columns go to the fragment
// slots of logical k = 4t..4t+3, its last four to 16+4t..16+4t+3.
//
// The level table (16 int8 levels per fp8 scale byte) is replicated 8 times
// with copy c living in bank group c; lane l reads copy l % 8, so the eight
// lanes of each quarter-warp phase of a 16-byte shared load never conflict.
//
// Grid: one CTA (8 warps) per 16 output rows; the warps split the K slices
// (s = warp, warp + 8, ...) and the int32 partial sums meet in shared memory.
#pragma once

#include "cr_device.cuh"

namespace cr {
namespace gv {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRows = 16;   // output rows per CTA
constexpr int kBatch = 4;   // slices whose loads are in flight together per warp

__device__ __forceinline__ void mma_s8(int32_t (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kThreads, 2)
    gemv_kernel(const int8_t *__restrict__ xq, const float *__restrict__ xs, const uint8_t *__restrict__ qdata,
                const uint8_t *__restrict__ srel, const float *__restrict__ codebook,
                const float *__restrict__ ws, const float *__restrict__ bias, int M, int64_t N, int64_t K,
                int out_f32, void *__restrict__ out, int32_t *__restrict__ acc_out)
{
    __shared__ uint4 lut8[256 * 8];  // lut8[s * 8 + c]: copy c of entry s
    __shared__ int32_t red[kWarps][kRows][8];
    __shared__ float cbs[16];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t n0 = (int64_t)blockIdx.x * kRows;
    const int64_t KH = K >> 1, KG = K >> 4;
    const int nslice = (int)(K >> 7);
    const int cnt = (nslice > warp) ? (nslice - warp + kWarps - 1) / kWarps : 0;

    const int64_t ra = n0 + g, rb = n0 + g + 8;
    const bool va = ra < N, vb = rb < N, vx = g < M;
    const uint8_t *pa = qdata + ra * KH + 16 * t;
    const uint8_t *pb = qdata + rb * KH + 16 * t;
    const uint8_t *psa = srel + ra * KG + 2 * t;
    const uint8_t *psb = srel + rb * KG + 2 * t;
    const int8_t *px = xq + (int64_t)g * K + 32 * t;
    const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);

    uint4 A[kBatch], B[kBatch], X0[kBatch], X1[kBatch];
    uint32_t SA[kBatch], SB[kBatch];

    // Weight loads (codes + group scales) and activation loads are issued
    // separately: the weights do not depend on the activation kernel, so they
    // can be in flight before griddepcontrol.wait.
    auto issue_w = [&](int i0) {
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = i0 + u;
            A[u] = B[u] = z4;
            SA[u] = SB[u] = 0u;
            if (i < cnt) {
                const int64_t s = warp + (int64_t)kWarps * i;
                if (va) {
                    A[u] = ldg_stream16(pa + 64 * s);
                    SA[u] = __ldg(reinterpret_cast<const uint16_t *>(psa + 8 * s));
                }
                if (vb) {
                    B[u] = ldg_stream16(pb + 64 * s);
                    SB[u] = __ldg(reinterpret_cast<const uint16_t *>(psb + 8 * s));
                }
            }
        }
    };
    auto issue_x = [&](int i0) {
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = i0 + u;
            X0[u] = X1[u] = z4;
            if (i < cnt && vx) {
                const int64_t s = warp + (int64_t)kWarps * i;
                X0[u] = *reinterpret_cast<const uint4 *>(px + 128 * s);
                X1[u] = *reinterpret_cast<const uint4 *>(px + 128 * s + 16);
            }
        }
    };

    // The first weight loads go out before the table is built, so its cost
    // hides under the memory latency.
    issue_w(0);

    if (tid < 16)
        cbs[tid] = codebook[tid];
    __syncthreads();
    {
        const uint4 e = lut_entry((uint32_t)tid, cbs);
#pragma unroll
        for (int r = 0; r < 8; ++r)
            lut8[tid * 8 + ((r + tid) & 7)] = e;
    }
    __syncthreads();

    // When launched as a programmatic dependent of the activation kernel, wait
    // here for its results (a no-op otherwise).
    asm volatile("griddepcontrol.wait;" ::: "memory");
    issue_x(0);

    int32_t c[4] = {0, 0, 0, 0};
    const int copy = lane & 7;
    for (int i0 = 0; i0 < cnt; i0 += kBatch) {
        if (i0 > 0) {
            issue_w(i0);
            issue_x(i0);
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (i0 + u < cnt) {
                const uint4 TA0 = lut8[(SA[u] & 0xFFu) * 8 + copy];
                const uint4 TA1 = lut8[(SA[u] >> 8) * 8 + copy];
                const uint4 TB0 = lut8[(SB[u] & 0xFFu) * 8 + copy];
                const uint4 TB1 = lut8[(SB[u] >> 8) * 8 + copy];
                uint32_t a0, a1, a2, a3;
                decode8(A[u].x, TA0, a0, a2);
                decode8(B[u].x, TB0, a1, a3);
                mma_s8(c, a0, a1, a2, a3, X0[u].x, X0[u].y);
                decode8(A[u].y, TA0, a0, a2);
                decode8(B[u].y, TB0, a1, a3);
                mma_s8(c, a0, a1, a2, a3, X0[u].z, X0[u].w);
                decode8(A[u].z, TA1, a0, a2);
                decode8(B[u].z, TB1, a1, a3);
                mma_s8(c, a0, a1, a2, a3, X1[u].x, X1[u].y);
                decode8(A[u].w, TA1, a0, a2);
                decode8(B[u].w, TB1, a1, a3);
                mma_s8(c, a0, a1, a2, a3, X1[u].z, X1[u].w);
            }
        }
    }

    // C fragment: c0 (row g, token 2t), c1 (g, 2t+1), c2 (g+8, 2t), c3 (g+8, 2t+1)
    red[warp][g][2 * t] = c[0];
    red[warp][g][2 * t + 1] = c[1];
    red[warp][g + 8][2 * t] = c[2];
    red[warp][g + 8][2 * t + 1] = c[3];
    __syncthreads();
    if (tid < kRows * 8) {
        const int r = tid >> 3, m = tid & 7;
        int32_t acc = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
            acc += red[w][r][m];
        const int64_t n = n0 + r;
        if (m < M && n < N) {
            const float y = epilogue_value(acc, xs[m], ws[n], bias, n);
            if (out_f32)
                reinterpret_cast<float *>(out)[(int64_t)m * N + n] = y;
            else
                reinterpret_cast<uint16_t *>(out)[(int64_t)m * N + n] = to_bf16_bits(y);
            if (acc_out != nullptr)
                acc_out[(int64_t)m * N + n] = acc;
        }
    }
}

// pdl: launch as a programmatic dependent of the previous kernel in the
// stream (the activation kernel), so the weight stream starts early.
inline cudaError_t launch(const int8_t *xq, const float *xs, const uint8_t *qdata, const uint8_t *srel,
                          const float *codebook, const float *ws, const float *bias, int64_t M, int64_t N, int64_t K,
                          int out_f32, void *out, int32_t *acc_out, cudaStream_t stream, bool pdl = false)
{
    const int64_t blocks = (N + kRows - 1) / kRows;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gemv_kernel, xq, xs, qdata, srel, codebook, ws, bias, (int)M, N, K, out_f32, out,
                              acc_out);
}

}  // namespace gv
}  // namespace cr
