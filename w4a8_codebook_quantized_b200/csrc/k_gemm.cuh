// k_gemm.cuh -- prefill contraction on the 5th-generation tensor cores.
//
// What it computes (ai-toolkit convrot_w4a8_quant.py, _w4a8_linear_ste_op:
// torch._int_mm(aq, w8.t()) followed by the epilogue):
//   acc[m, n] = sum_k A[m, k] * B[n, k]   A = xq [M, K] int8, B = w8 [N, K] int8
//   out[m, n] = float(acc) * (xs[m] * ws[n]) [+ bias[n]]
//
// B200 design: a persistent, warp-specialised kernel, one CTA per SM.
//   warp 0      one thread issues TMA loads of 128-wide K slices of the A tile
//               (128 rows) and the B tile (256 rows) into a 4-stage ring of
//               128-byte-swizzled shared-memory buffers (48 KB per stage);
//   warp 1      allocates 512 TMEM columns (two 128 x 256 int32 accumulators)
//               and one thread issues tcgen05.mma kind::i8 (M 128, N 256, K 32,
//               four per stage), releasing each stage with tcgen05.commit;
//   warps 2-5   the epilogue: tcgen05.ld of 32 columns at a time, the
//               per-token x per-channel fp32 rescale (+ bias), bf16 or fp32
//               stores, then the TMEM buffer is handed back to the MMA warp,
//               so the epilogue of tile i overlaps the MMAs of tile i + 1.
// Every wait is bounded (a second or two); a wait that runs out sets the
// library error word, every role stops, TMEM is freed and the kernel returns.
// TMA zero-fills rows past M or N, so ragged edges need no special casing
// except in the epilogue's stores.
#pragma once

#include <cuda.h>

#include <type_traits>

#include "cr_device.cuh"

namespace cr {
namespace gm {

constexpr int BM = 128, BN = 256, BK = 128;  // BK in int8 elements = bytes
constexpr int kStages = 4;
constexpr int kABytes = BM * BK;              // 16 KB
constexpr int kBBytes = BN * BK;              // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kTmemCols = 2 * BN;             // two accumulators
constexpr int kThreads = 192;
constexpr uint32_t kIdesc = idesc_i8(BM, BN);

constexpr int kEpiBytes = 32 * 128;  // one epilogue store unit: 32 rows x 128 bytes

struct __align__(1024) Smem {
    uint8_t stage[kStages][kStageBytes];  // A at +0, B at +kABytes; every buffer 1024-aligned
    uint8_t epi[4][kEpiBytes];            // per epilogue warp, one 128B-swizzled staging unit
    float wsb[2][BN];                     // per-tile channel scales (double-buffered by tile parity)
    float biasb[2][BN];                   // per-tile bias
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint32_t tmem_base;
    int abort;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;  // + slack to align the base

__device__ __forceinline__ void tile_coords(int tile, int tiles_n, int &tm, int &tn)
{
    tm = tile / tiles_n;
    tn = tile - tm * tiles_n;
}

// Epilogue of one 128 x 256 accumulator tile for one warp: its 32 TMEM lanes
// are rows row0 + lane; `tbase` addresses lane 0 of the warp's quarter at the
// tile's first column; the output columns are col_base + [0, 256).  Fast path
// (tma_out): 128-byte column units (64 bf16 or 32 fp32 columns) go through the
// 128B-swizzled staging buffer `stage_buf` (16-byte chunk c of row r at chunk
// c ^ (r % 8): conflict-free) and one TMA bulk store each; the next 32-column
// TMEM load is in flight while the current chunk is converted.  Otherwise each
// thread stores its own row.  release() hands the accumulator back once every
// column is in registers.
// RAW: the accumulator holds fp32 values that are the outputs themselves
// (bf16 GEMM); no scales, bias or SwiGLU.
template <bool RAW, class Release>
__device__ __forceinline__ void epilogue_tile(uint32_t tbase, int row0, int col_base, int lane, float xm, bool row_ok,
                                              const float *wsv, const float *bsv, bool has_bias, int M, int N,
                                              int out_f32, int swiglu, int tma_out, const CUtensorMap *tmOut,
                                              uint8_t *stage_buf,
                                              uint32_t &units_issued, void *__restrict__ out,
                                              int32_t *__restrict__ acc_out, const float *__restrict__ ws,
                                              const float *__restrict__ bias, Release release)
{
    const int row = row0 + lane;
    // 32 accumulators of columns [c0, c0 + 32) of the tile -> 32 fp32 or 16 bf16x2 words
    auto convert32 = [&](const uint32_t (&v)[32], int c0, uint32_t *dst) {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
            float y[4];
            if constexpr (RAW) {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    y[e] = __uint_as_float(v[j + e]);
            } else {
                const float4 w4 = *reinterpret_cast<const float4 *>(wsv + c0 + j);
                const float4 b4 = *reinterpret_cast<const float4 *>(bsv + c0 + j);
                const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
                const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    y[e] = __fmul_rn(__int2float_rn((int32_t)v[j + e]), __fmul_rn(xm, wv[e]));
                    if (has_bias)
                        y[e] = __fadd_rn(y[e], bv[e]);
                }
            }
            if (out_f32) {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    dst[j + e] = __float_as_uint(y[e]);
            } else {
                dst[j / 2] = to_bf16x2_bits(y[0], y[1]);
                dst[j / 2 + 1] = to_bf16x2_bits(y[2], y[3]);
            }
        }
    };
    // one 128-byte unit of the warp's 32 rows -> staging buffer -> TMA bulk store
    auto store_unit = [&](const uint32_t (&p)[32], int ucol0) {
        if (units_issued >= 1) {
            if (lane == 0)
                bulk_wait_read<0>();  // the previous store has read the staging buffer
            __syncwarp();
        }
        uint8_t *stg = stage_buf;
#pragma unroll
        for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4 *>(stg + lane * 128 + ((c ^ (lane & 7)) * 16)) =
                make_uint4(p[4 * c], p[4 * c + 1], p[4 * c + 2], p[4 * c + 3]);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(tmOut, ucol0, row0, stg);
            bulk_commit();
        }
        ++units_issued;
    };
    uint32_t cur[32], nxt[32], packed[32];
    if (!RAW && swiglu) {
        // Interleaved gate/up rows: accumulator columns 2f and 2f + 1 are one
        // pair and give output column f of [M, N / 2].  Each 32-column TMEM
        // load yields 16 outputs; a 128-byte unit (64 bf16 or 32 fp32 outputs)
        // takes 4 or 2 loads.
        const int F = N >> 1, ocol_base = col_base >> 1;
        auto pairs16 = [&](int c0, float (&y)[16]) {
#pragma unroll
            for (int p = 0; p < 16; ++p) {
                float g = __fmul_rn(__int2float_rn((int32_t)cur[2 * p]), __fmul_rn(xm, wsv[c0 + 2 * p]));
                float u = __fmul_rn(__int2float_rn((int32_t)cur[2 * p + 1]), __fmul_rn(xm, wsv[c0 + 2 * p + 1]));
                if (has_bias) {
                    g = __fadd_rn(g, bsv[c0 + 2 * p]);
                    u = __fadd_rn(u, bsv[c0 + 2 * p + 1]);
                }
                y[p] = swiglu_value(g, u);
            }
        };
        // uo: output columns per 128-byte unit (compile-time, so that `packed`
        // stays in registers)
        auto units = [&](auto uo_c) {
            constexpr int uo = decltype(uo_c)::value;
            for (int un = 0; un < BN / (2 * uo); ++un) {
#pragma unroll
                for (int k = 0; k < uo / 16; ++k) {
                    const int c0 = 2 * uo * un + 32 * k;
                    __syncwarp();
                    tmem_ld_32cols(tbase + (uint32_t)c0, cur);
                    tmem_ld_wait();
                    if (c0 + 32 == BN)
                        release();
                    float y[16];
                    pairs16(c0, y);
                    if constexpr (uo == 32) {
#pragma unroll
                        for (int p = 0; p < 16; ++p)
                            packed[16 * k + p] = __float_as_uint(y[p]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            packed[8 * k + i] = to_bf16x2_bits(y[2 * i], y[2 * i + 1]);
                    }
                }
                store_unit(packed, ocol_base + uo * un);
            }
        };
        if (tma_out && out_f32) {
            units(std::integral_constant<int, 32>{});
        } else if (tma_out) {
            units(std::integral_constant<int, 64>{});
        } else {
            for (int ch = 0; ch < BN / 32; ++ch) {
                const int c0 = 32 * ch;
                __syncwarp();
                tmem_ld_32cols(tbase + (uint32_t)c0, cur);
                tmem_ld_wait();
                if (ch + 1 == BN / 32)
                    release();
                float y[16];
                pairs16(c0, y);
                const int f0 = ocol_base + 16 * ch;
                if (row_ok && f0 < F) {
                    const int64_t base = (int64_t)row * F + f0;
#pragma unroll
                    for (int p = 0; p < 16; ++p) {
                        if (f0 + p >= F)
                            break;
                        if (out_f32)
                            reinterpret_cast<float *>(out)[base + p] = y[p];
                        else
                            reinterpret_cast<uint16_t *>(out)[base + p] = to_bf16_bits(y[p]);
                    }
                }
            }
        }
        return;
    }
    __syncwarp();
    tmem_ld_32cols(tbase, cur);
    tmem_ld_wait();
    if (tma_out && !out_f32) {
        // units of 64 columns: two 32-column chunks each
        for (int u = 0; u < BN / 64; ++u) {
            __syncwarp();
            tmem_ld_32cols(tbase + (uint32_t)(64 * u + 32), nxt);
            convert32(cur, 64 * u, packed);
            tmem_ld_wait();
            if (u + 1 < BN / 64) {
                __syncwarp();
                tmem_ld_32cols(tbase + (uint32_t)(64 * u + 64), cur);
            } else {
                release();
            }
            convert32(nxt, 64 * u + 32, packed + 16);
            store_unit(packed, col_base + 64 * u);
            if (u + 1 < BN / 64)
                tmem_ld_wait();
        }
    } else if (tma_out) {
        // units of 32 fp32 columns
        for (int u = 0; u < BN / 32; ++u) {
            if (u + 1 < BN / 32) {
                __syncwarp();
                tmem_ld_32cols(tbase + (uint32_t)(32 * u + 32), nxt);
            } else {
                release();
            }
            convert32(cur, 32 * u, packed);
            store_unit(packed, col_base + 32 * u);
            if (u + 1 < BN / 32) {
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    cur[j] = nxt[j];
            }
        }
    } else {
        for (int ch = 0; ch < BN / 32; ++ch) {
            if (ch + 1 < BN / 32) {
                __syncwarp();
                tmem_ld_32cols(tbase + (uint32_t)(32 * (ch + 1)), nxt);
            } else {
                release();
            }
            const int col0 = col_base + 32 * ch;
            if (row_ok && col0 < N) {
                const int64_t base = (int64_t)row * N + col0;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int n = col0 + j;
                    if (n >= N)
                        break;
                    const float y = RAW ? __uint_as_float(cur[j]) : epilogue_value((int32_t)cur[j], xm, ws[n], bias, n);
                    if (out_f32)
                        reinterpret_cast<float *>(out)[base + j] = y;
                    else
                        reinterpret_cast<uint16_t *>(out)[base + j] = to_bf16_bits(y);
                    if (acc_out != nullptr)
                        acc_out[base + j] = (int32_t)cur[j];
                }
            }
            if (ch + 1 < BN / 32) {
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    cur[j] = nxt[j];
            }
        }
    }
}

// BF16: A and B are bf16 (K counted in bf16 elements, 64 per 128-byte
// stage row), tcgen05.mma kind::f16 into fp32, and the epilogue writes the
// accumulators as they are (xs, ws, bias, swiglu and acc_out unused).
template <bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmOut, const float *__restrict__ xs,
                const float *__restrict__ ws, const float *__restrict__ bias, int M, int N, int K, int out_f32,
                int swiglu, int tma_out, void *__restrict__ out, int32_t *__restrict__ acc_out)
{
    extern __shared__ uint8_t smem_raw[];
    Smem &sh = smem_aligned_1024<Smem>(smem_raw);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_m = (M + BM - 1) / BM, tiles_n = (N + BN - 1) / BN;
    const int num_tiles = tiles_m * tiles_n;
    constexpr int BKE = BF16 ? BK / 2 : BK;  // K elements per stage
    const int kblocks = (K + BKE - 1) / BKE;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sh.tmem_full[b], 1);
            mbar_init(&sh.tmem_empty[b], 4);
        }
        sh.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        tmem_alloc(&sh.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    volatile int *abort = &sh.abort;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmA);
            prefetch_tmap(&tmB);
            int stage = 0;
            uint32_t phase = 0;
            int issued[kStages];
            uint32_t issued_phase[kStages];
            for (int s = 0; s < kStages; ++s)
                issued[s] = 0, issued_phase[s] = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                int tm, tn;
                tile_coords(tile, tiles_n, tm, tn);
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait_bounded(&sh.empty[stage], phase ^ 1u, abort)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sh.full[stage], kStageBytes);
                    tma_load_2d(sh.stage[stage], &tmA, kb * BKE, tm * BM, &sh.full[stage]);
                    tma_load_2d(sh.stage[stage] + kABytes, &tmB, kb * BKE, tn * BN, &sh.full[stage]);
                    issued[stage] = 1;
                    issued_phase[stage] = phase;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // Let copies already in flight land before the CTA goes away.
                for (int s = 0; s < kStages; ++s)
                    if (issued[s]) {
                        volatile int no_abort = 0;
                        mbar_wait_bounded(&sh.full[s], issued_phase[s], &no_abort, 20000000ull);
                    }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int local = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++local) {
                const int buf = local & 1;
                const uint32_t use = (uint32_t)(local >> 1) & 1u;
                if (!mbar_wait_bounded(&sh.tmem_empty[buf], use ^ 1u, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(buf * BN);
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait_bounded(&sh.full[stage], phase, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(sh.stage[stage]);
                    const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk) {
                        const uint64_t ad = sw128_kmajor_desc(a_addr + 32u * kk);
                        const uint64_t bd = sw128_kmajor_desc(b_addr + 32u * kk);
                        if constexpr (BF16)
                            mma_bf16(d, ad, bd, idesc_bf16(BM, BN), (kb | kk) != 0 ? 1u : 0u);
                        else
                            mma_i8(d, ad, bd, kIdesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit(&sh.empty[stage]);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok)
                    tc_commit(&sh.tmem_full[buf]);
            }
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2..5)
        // Warp q owns TMEM lanes 32q..32q+31 = rows 32q.. of the tile.
        // Per tile: the 128 epilogue threads stage the tile's channel scales
        // (and bias) in shared memory before waiting for the accumulator, so
        // that latency hides under the MMAs.  The accumulator is read 32
        // columns at a time, the next chunk's TMEM load in flight while the
        // current one is converted.  Fast path (tma_out): each 128-byte column
        // unit (64 bf16 or 32 fp32 columns) of the warp's 32 rows goes into a
        // 128B-swizzled staging buffer (16-byte chunk c of row r at chunk
        // c ^ (r % 8): conflict-free) and leaves with one TMA bulk store.  Otherwise (int32 accumulators requested, or rows
        // not 16-byte multiples) each thread stores its own row.
        // The loop never exits early: after an abort every warp still reaches
        // the same named barriers, skipping the work.
        const int q = warp & 3;
        const int et = threadIdx.x - 64;  // 0..127 among the epilogue threads
        int local = 0;
        uint32_t units_issued = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
            int tm, tn;
            tile_coords(tile, tiles_n, tm, tn);
            const int buf = local & 1;
            const uint32_t use = (uint32_t)(local >> 1) & 1u;
            if constexpr (!BF16) {
                for (int j = et; j < BN; j += 128) {
                    const int n = tn * BN + j;
                    sh.wsb[buf][j] = n < N ? ws[n] : 0.0f;
                    sh.biasb[buf][j] = (bias != nullptr && n < N) ? bias[n] : 0.0f;
                }
            }
            asm volatile("bar.sync 2, 128;" ::: "memory");
            const bool ok = mbar_wait_bounded_warp(&sh.tmem_full[buf], use, abort);
            if (!ok)
                continue;
            tc_fence_after();
            const int row = tm * BM + 32 * q + lane;
            const bool row_ok = row < M;
            const float xm = (!BF16 && row_ok) ? xs[row] : 0.0f;
            const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * BN);
            epilogue_tile<BF16>(tbase, tm * BM + 32 * q, tn * BN, lane, xm, row_ok, sh.wsb[buf], sh.biasb[buf],
                          bias != nullptr, M, N, out_f32, swiglu, tma_out, &tmOut, sh.epi[q], units_issued, out, acc_out, ws,
                          bias, [&]() {
                              tc_fence_before();
                              __syncwarp();
                              if (lane == 0)
                                  mbar_arrive(&sh.tmem_empty[buf]);
                          });
        }
        if (lane == 0)
            bulk_wait_all();  // every output store has landed before the CTA exits
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}


// ---------------------------------------------------------------- CTA-pair variant
//
// For problems with at least one 256 x 256 tile per SM pair: a cluster of two
// CTAs computes a 256 x 256 tile with tcgen05.mma.cta_group::2 (M = 256,
// N = 256, K = 32).  Each CTA loads only its own 128 rows of A and its own 128
// rows of B (no multicast loads), so every SM moves 32 KB instead of 48 KB per
// 128-wide K slice for the same MMA work; each CTA's TMEM receives its 128 rows
// of the accumulator.  The leader (rank 0) issues the MMAs; both CTAs' TMA
// copies signal the leader's "full" barrier; the leader's commits are sent to
// both CTAs' "empty" and "tmem_full" barriers; both CTAs' epilogue warps
// release the accumulator on the leader's "tmem_empty" barrier.
namespace pair {
constexpr int kStages = 6;
constexpr int kHalfBytes = 128 * BK;           // 16 KB: one CTA's half of A or of B
constexpr int kStageBytes = 2 * kHalfBytes;    // A half at +0, B half at +16 KB
constexpr uint32_t kIdesc = idesc_i8(256, BN);

struct __align__(1024) Smem {
    uint8_t stage[kStages][kStageBytes];
    uint8_t epi[4][kEpiBytes];
    float wsb[2][BN];
    float biasb[2][BN];
    uint64_t full[kStages];       // leader: both CTAs' bytes of a stage
    uint64_t empty[kStages];      // each CTA: its stage may be refilled
    uint64_t tmem_full[2];        // each CTA: its accumulator rows are complete
    uint64_t tmem_empty[2];       // leader: both CTAs' epilogues released the accumulator
    uint32_t tmem_base;
    int abort;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
}  // namespace pair

// BF16 as for gemm_kernel.
template <bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmOut, const float *__restrict__ xs,
                     const float *__restrict__ ws, const float *__restrict__ bias, int M, int N, int K, int out_f32,
                     int swiglu, int tma_out, void *__restrict__ out, int32_t *__restrict__ acc_out)
{
    extern __shared__ uint8_t smem_raw[];
    pair::Smem &sh = smem_aligned_1024<pair::Smem>(smem_raw);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int npairs = gridDim.x >> 1, pair_id = blockIdx.x >> 1;
    const int tiles_m = (M + 255) / 256, tiles_n = (N + BN - 1) / BN;
    const int num_tiles = tiles_m * tiles_n;
    constexpr int BKE = BF16 ? BK / 2 : BK;  // K elements per stage
    const int kblocks = (K + BKE - 1) / BKE;

    if (threadIdx.x == 0) {
        for (int s = 0; s < pair::kStages; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sh.tmem_full[b], 1);
            mbar_init(&sh.tmem_empty[b], 8);
        }
        sh.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        tmem_alloc_pair(&sh.tmem_base, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers exist before anyone signals them
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    volatile int *abort = &sh.abort;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            prefetch_tmap(&tmA);
            prefetch_tmap(&tmB);
            int stage = 0;
            uint32_t phase = 0;
            int issued[pair::kStages];
            uint32_t issued_phase[pair::kStages];
            for (int s = 0; s < pair::kStages; ++s)
                issued[s] = 0, issued_phase[s] = 0;
            bool ok = true;
            for (int tile = pair_id; ok && tile < num_tiles; tile += npairs) {
                int tm, tn;
                tile_coords(tile, tiles_n, tm, tn);
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait_bounded(&sh.empty[stage], phase ^ 1u, abort)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full_leader = mapa_shared(smem_u32(&sh.full[stage]), 0);
                    if (leader)
                        mbar_arrive_expect_tx(&sh.full[stage], 2 * pair::kStageBytes);
                    tma_load_2d_pair(sh.stage[stage], &tmA, kb * BKE, tm * 256 + (int)rank * 128, full_leader);
                    tma_load_2d_pair(sh.stage[stage] + pair::kHalfBytes, &tmB, kb * BKE, tn * BN + (int)rank * 128,
                                     full_leader);
                    issued[stage] = 1;
                    issued_phase[stage] = phase;
                    if (++stage == pair::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // let copies in flight land before the CTAs go away: the leader
                // waits on its barriers (bounded); the partner, whose copies
                // signal the leader, waits a fixed 100 us
                if (leader) {
                    for (int s = 0; s < pair::kStages; ++s)
                        if (issued[s]) {
                            volatile int no_abort = 0;
                            mbar_wait_bounded(&sh.full[s], issued_phase[s], &no_abort, 20000000ull);
                        }
                } else {
                    const uint64_t t0 = globaltimer_ns();
                    while (globaltimer_ns() - t0 < 100000ull) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader only)
        if (leader && lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int local = 0;
            bool ok = true;
            const uint32_t peer = 1;
            for (int tile = pair_id; ok && tile < num_tiles; tile += npairs, ++local) {
                const int buf = local & 1;
                const uint32_t use = (uint32_t)(local >> 1) & 1u;
                if (!mbar_wait_bounded(&sh.tmem_empty[buf], use ^ 1u, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(buf * BN);
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait_bounded(&sh.full[stage], phase, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(sh.stage[stage]);
                    const uint32_t b_addr = a_addr + pair::kHalfBytes;
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk)
                        if constexpr (BF16)
                            mma_bf16_pair(d, sw128_kmajor_desc(a_addr + 32u * kk),
                                          sw128_kmajor_desc(b_addr + 32u * kk), idesc_bf16(256, BN),
                                          (kb | kk) != 0 ? 1u : 0u);
                        else
                            mma_i8_pair(d, sw128_kmajor_desc(a_addr + 32u * kk),
                                        sw128_kmajor_desc(b_addr + 32u * kk), pair::kIdesc,
                                        (kb | kk) != 0 ? 1u : 0u);
                    const uint32_t e = smem_u32(&sh.empty[stage]);
                    tc_commit_pair(mapa_shared(e, 0));
                    tc_commit_pair(mapa_shared(e, peer));
                    if (++stage == pair::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) {
                    const uint32_t f = smem_u32(&sh.tmem_full[buf]);
                    tc_commit_pair(mapa_shared(f, 0));
                    tc_commit_pair(mapa_shared(f, peer));
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2..5, both CTAs)
        const int q = warp & 3;
        const int et = threadIdx.x - 64;
        int local = 0;
        uint32_t units_issued = 0;
        for (int tile = pair_id; tile < num_tiles; tile += npairs, ++local) {
            int tm, tn;
            tile_coords(tile, tiles_n, tm, tn);
            const int buf = local & 1;
            const uint32_t use = (uint32_t)(local >> 1) & 1u;
            if constexpr (!BF16) {
                for (int j = et; j < BN; j += 128) {
                    const int n = tn * BN + j;
                    sh.wsb[buf][j] = n < N ? ws[n] : 0.0f;
                    sh.biasb[buf][j] = (bias != nullptr && n < N) ? bias[n] : 0.0f;
                }
            }
            asm volatile("bar.sync 2, 128;" ::: "memory");
            const bool ok = mbar_wait_bounded_warp(&sh.tmem_full[buf], use, abort);
            if (!ok)
                continue;
            tc_fence_after();
            const int row0 = tm * 256 + (int)rank * 128 + 32 * q;
            const bool row_ok = row0 + lane < M;
            const float xm = (!BF16 && row_ok) ? xs[row0 + lane] : 0.0f;
            const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * BN);
            const uint32_t release_addr = mapa_shared(smem_u32(&sh.tmem_empty[buf]), 0);
            epilogue_tile<BF16>(tbase, row0, tn * BN, lane, xm, row_ok, sh.wsb[buf], sh.biasb[buf], bias != nullptr, M,
                          N, out_f32, swiglu, tma_out, &tmOut, sh.epi[q], units_issued, out, acc_out, ws, bias, [&]() {
                              tc_fence_before();
                              __syncwarp();
                              if (lane == 0)
                                  mbar_arrive_cluster(release_addr);
                          });
        }
        if (lane == 0)
            bulk_wait_all();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // no CTA leaves while its partner may still signal it
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

}  // namespace gm
}  // namespace cr
