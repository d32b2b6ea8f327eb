// k_gemv.cuh -- fused decode GEMV for M <= 8 tokens.
//
// What it computes (ai-toolkit convrot_w4a8_quant.py, w4a8_gemv_kernel):
// out[m, n] = epilogue(sum_k xq[m, k] * w8[n, k]) with w8 decoded on the fly
// from the packed codes, the fp8 group scales and the codebook, so the weight
// costs 4.5 bits of HBM traffic and is never materialised.  The int32 sums
// are exact, so the result equals the prefill path bit for bit.
//
// B200 design.
//  * Streaming: a persistent grid (several CTAs per SM).  In each CTA one
//    producer warp moves tiles of 16 weight rows x 1024 columns of the packed
//    codes (8 KB) and their group scales (1 KB) into a ring of shared-memory
//    stages with 2-D TMA copies; eight consumer warps decode and contract each
//    stage while the following ones are in flight.  Bytes in flight are set by the
//    ring, not by registers, which keeps HBM busy.
//  * Decode: a per-CTA table of the 16 int8 levels of every fp8 scale byte
//    (exact: the decoded value depends only on the pair), replicated 8 times
//    with copy c in bank group c so that a quarter-warp's 16-byte lookups
//    never conflict; byte permutes turn 8 packed codes into 8 int8 levels.
//  * Contraction: the page's kernel uses int32 IMAD in registers; here the
//    decoded weights go straight from registers into the warp-level int8
//    tensor-core instruction (mma.sync m16n8k32: A = 16 weight rows x 32 k,
//    B = 32 k x 8 tokens), so the ALU only pays for the decode.  Since the sum
//    runs over k, any permutation of k is allowed as long as A and B use the
//    same one: thread (g = lane / 4, t = lane % 4) takes the 16 contiguous
//    bytes (32 codes) of rows g and g + 8 at k = 128 w + 32 t of its warp's
//    slice w, and the matching 32 activation bytes of token g; code word i
//    (columns 8i..8i+7) feeds MMA i, its first four columns in the fragment
//    slots of logical k = 4t..4t+3 and its last four in 16+4t..16+4t+3.
//  * The int32 partial sums of the eight warps meet in shared memory; the
//    fused epilogue writes the 16 x M outputs of the row tile.
//  * When launched as a programmatic dependent of the activation kernel, the
//    weight stream and the table build start before that kernel finishes;
//    the consumers wait for it (griddepcontrol.wait) before reading xq / xs.
#pragma once

#include <cuda.h>

#include "cr_device.cuh"

namespace cr {
namespace gv {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;  // + one producer warp

// Shape of the pipeline.  A tile is RG groups of 16 weight rows; every
// consumer warp takes SLICES slices of 128 k per stage, so a stage covers
// CHUNK = 8 * SLICES * 128 columns of the tile's 16 RG rows.  MINB is the
// number of CTAs the kernel is compiled to fit on one SM.
template <int RG, int SLICES, int STAGES, int MINB>
struct Cfg {
    static constexpr int kRG = RG;
    static constexpr int kRows = 16 * RG;
    static constexpr int kSlices = SLICES;
    static constexpr int kStages = STAGES;
    static constexpr int kMinBlocks = MINB;
    static constexpr int kChunk = kConsumerWarps * SLICES * 128;
    static constexpr int kCodeBytes = kRows * kChunk / 2;
    static constexpr int kSrelBytes = kRows * kChunk / 16;
    struct __align__(1024) Smem {
        uint8_t codes[STAGES][kCodeBytes];  // row r of a stage at r * kChunk / 2 bytes
        uint8_t srel[STAGES][kSrelBytes];   // row r of a stage at r * kChunk / 16 bytes
        uint4 lut8[256 * 8];                // lut8[s * 8 + c]: copy c of the levels of scale byte s
        int32_t red[kConsumerWarps][kRows][8];
        float cb[16];
        uint64_t full[STAGES];
        uint64_t empty[STAGES];
        int abort;
    };
    static constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
};

// The configuration the library launches.
using Prod = Cfg<1, 1, 4, 3>;

__device__ __forceinline__ void mma_s8(int32_t (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// One slice of one 16-row group: rows g and g + 8 (relative to the group) x
// 128 k of this stage against the token fragments X0, X1.  `lutc` already
// points at this lane's table copy; entry s is lutc[8 s].
__device__ __forceinline__ void slice_mma(const uint8_t *codes_g, const uint8_t *codes_g8, const uint8_t *srel_g,
                                          const uint8_t *srel_g8, const uint4 *lutc, const uint4 &X0,
                                          const uint4 &X1, int32_t (&c)[4], int32_t (&d)[4])
{
    const uint4 A = *reinterpret_cast<const uint4 *>(codes_g);
    const uint4 B = *reinterpret_cast<const uint4 *>(codes_g8);
    const uint4 TA0 = lutc[8 * (uint32_t)srel_g[0]];
    const uint4 TA1 = lutc[8 * (uint32_t)srel_g[1]];
    const uint4 TB0 = lutc[8 * (uint32_t)srel_g8[0]];
    const uint4 TB1 = lutc[8 * (uint32_t)srel_g8[1]];
    uint32_t a0, a1, a2, a3, e0, e1, e2, e3;
    decode8(A.x, TA0, a0, a2);
    decode8(B.x, TB0, a1, a3);
    decode8(A.y, TA0, e0, e2);
    decode8(B.y, TB0, e1, e3);
    mma_s8(c, a0, a1, a2, a3, X0.x, X0.y);
    mma_s8(d, e0, e1, e2, e3, X0.z, X0.w);
    decode8(A.z, TA1, a0, a2);
    decode8(B.z, TB1, a1, a3);
    decode8(A.w, TA1, e0, e2);
    decode8(B.w, TB1, e1, e3);
    mma_s8(c, a0, a1, a2, a3, X1.x, X1.y);
    mma_s8(d, e0, e1, e2, e3, X1.z, X1.w);
}

template <class C>
__global__ void __launch_bounds__(kThreads, C::kMinBlocks)
    gemv_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_srel,
                const int8_t *__restrict__ xq, const float *__restrict__ xs, const float *__restrict__ codebook,
                const float *__restrict__ ws, const float *__restrict__ bias, int M, int N, int K, int out_f32,
                void *__restrict__ out, int32_t *__restrict__ acc_out)
{
    constexpr int RG = C::kRG, ROWS = C::kRows, S = C::kSlices, STAGES = C::kStages, CHUNK = C::kChunk;
    using Smem = typename C::Smem;
    extern __shared__ uint8_t smem_raw[];
    Smem &sh = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ntiles = (N + ROWS - 1) / ROWS;
    const int nchunks = (K + CHUNK - 1) / CHUNK;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], kConsumerWarps);
        }
        sh.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (tid < 16)
        sh.cb[tid] = codebook[tid];
    __syncthreads();
    volatile int *abort = &sh.abort;

    if (warp == kConsumerWarps) {
        // ------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tm_codes);
            prefetch_tmap(&tm_srel);
            int stage = 0;
            uint32_t phase = 0;
            int issued[STAGES];
            uint32_t issued_phase[STAGES];
            for (int s = 0; s < STAGES; ++s)
                issued[s] = 0, issued_phase[s] = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
                for (int c = 0; c < nchunks; ++c) {
                    if (!mbar_wait_bounded(&sh.empty[stage], phase ^ 1u, abort)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sh.full[stage], C::kCodeBytes + C::kSrelBytes);
                    tma_load_2d(sh.codes[stage], &tm_codes, c * (CHUNK / 8), tile * ROWS, &sh.full[stage]);
                    tma_load_2d(sh.srel[stage], &tm_srel, c * (CHUNK / 16), tile * ROWS, &sh.full[stage]);
                    issued[stage] = 1;
                    issued_phase[stage] = phase;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                for (int s = 0; s < STAGES; ++s)
                    if (issued[s]) {
                        volatile int no_abort = 0;
                        mbar_wait_bounded(&sh.full[s], issued_phase[s], &no_abort, 20000000ull);
                    }
            }
        }
    } else {
        // ------------------------------------------------ consumers
        {
            const uint4 e = lut_entry((uint32_t)tid, sh.cb);
#pragma unroll
            for (int r = 0; r < 8; ++r)
                sh.lut8[tid * 8 + ((r + tid) & 7)] = e;
        }
        consumer_sync();
        asm volatile("griddepcontrol.wait;" ::: "memory");

        const int g = lane >> 2, t = lane & 3;
        const uint4 *lutc = sh.lut8 + (lane & 7);
        const bool vx = g < M;
        // slice j of this warp in a stage: k offset 128 * (warp + 8 j) in the chunk
        const int8_t *px = xq + (int64_t)g * K + 128 * warp + 32 * t;
        const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
        // The activation fragments of a chunk do not depend on the row tile;
        // the next chunk's are fetched (through L1/L2) while the current one
        // is computed.  Two register sets alternate with the chunk parity.
        auto fetch_x = [&](int ch, uint4 (&X)[S][2]) {
#pragma unroll
            for (int j = 0; j < S; ++j) {
                X[j][0] = X[j][1] = z4;
                const int k0 = ch * CHUNK + 128 * (warp + 8 * j);
                if (vx && k0 < K) {
                    X[j][0] = *reinterpret_cast<const uint4 *>(px + (int64_t)ch * CHUNK + 1024 * j);
                    X[j][1] = *reinterpret_cast<const uint4 *>(px + (int64_t)ch * CHUNK + 1024 * j + 16);
                }
            }
        };
        uint4 XA[S][2], XB[S][2];
        int stage = 0;
        uint32_t phase = 0;
        // consume one stage: all slices of this warp, all row groups
        auto consume = [&](int ch, const uint4 (&X)[S][2], int32_t (&c)[RG][4], int32_t (&d)[RG][4]) {
            const bool ok = mbar_wait_bounded_warp(&sh.full[stage], phase, abort);
            if (ok) {
#pragma unroll
                for (int j = 0; j < S; ++j) {
                    const int sl = warp + 8 * j;
                    if (ch * CHUNK + 128 * sl < K) {
                        const uint8_t *cs = sh.codes[stage] + 64 * sl + 16 * t + (CHUNK / 2) * g;
                        const uint8_t *ss = sh.srel[stage] + 8 * sl + 2 * t + (CHUNK / 16) * g;
#pragma unroll
                        for (int rg = 0; rg < RG; ++rg)
                            slice_mma(cs + (CHUNK / 2) * 16 * rg, cs + (CHUNK / 2) * (16 * rg + 8),
                                      ss + (CHUNK / 16) * 16 * rg, ss + (CHUNK / 16) * (16 * rg + 8), lutc,
                                      X[j][0], X[j][1], c[rg], d[rg]);
                    }
                }
            }
            __syncwarp();
            if (ok && lane == 0)
                mbar_arrive(&sh.empty[stage]);
            if (++stage == STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        };
        fetch_x(0, XA);
        int xnext = nchunks > 1 ? 1 : 0;  // chunk whose fragments are fetched next
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
            // two accumulators per row group break the dependency chain between MMAs
            int32_t c[RG][4], d[RG][4];
#pragma unroll
            for (int rg = 0; rg < RG; ++rg)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    c[rg][i] = d[rg][i] = 0;
            // chunks in pairs: XA holds the even chunk's fragments, XB the odd one's
            for (int ch = 0; ch < nchunks; ch += 2) {
                fetch_x(xnext, XB);
                if (++xnext == nchunks)
                    xnext = 0;
                consume(ch, XA, c, d);
                if (ch + 1 < nchunks) {
                    fetch_x(xnext, XA);
                    if (++xnext == nchunks)
                        xnext = 0;
                    consume(ch + 1, XB, c, d);
                } else {
                    // odd chunk count: XB holds the next tile's chunk 0
#pragma unroll
                    for (int j = 0; j < S; ++j)
                        XA[j][0] = XB[j][0], XA[j][1] = XB[j][1];
                }
            }
#pragma unroll
            for (int rg = 0; rg < RG; ++rg) {
                // C fragment: c0 (row g, token 2t), c1 (g, 2t+1), c2 (g+8, 2t), c3 (g+8, 2t+1)
                sh.red[warp][16 * rg + g][2 * t] = c[rg][0] + d[rg][0];
                sh.red[warp][16 * rg + g][2 * t + 1] = c[rg][1] + d[rg][1];
                sh.red[warp][16 * rg + g + 8][2 * t] = c[rg][2] + d[rg][2];
                sh.red[warp][16 * rg + g + 8][2 * t + 1] = c[rg][3] + d[rg][3];
            }
            consumer_sync();
            for (int e = tid; e < ROWS * 8; e += 256) {
                const int r = e >> 3, m = e & 7;
                int32_t acc = 0;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w)
                    acc += sh.red[w][r][m];
                const int n = tile * ROWS + r;
                if (m < M && n < N && !*abort) {
                    const float y = epilogue_value(acc, xs[m], ws[n], bias, n);
                    const int64_t o = (int64_t)m * N + n;
                    if (out_f32)
                        reinterpret_cast<float *>(out)[o] = y;
                    else
                        reinterpret_cast<uint16_t *>(out)[o] = to_bf16_bits(y);
                    if (acc_out != nullptr)
                        acc_out[o] = acc;
                }
            }
            consumer_sync();
        }
    }
    __syncthreads();
}

}  // namespace gv
}  // namespace cr
