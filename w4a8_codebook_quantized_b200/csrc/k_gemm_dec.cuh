// k_gemm_dec.cuh -- prefill contraction with the weight decode fused into the
// producer side of the CTA-pair tcgen05 GEMM.
//
// What it computes is gm::gemm_pair_kernel's result (ai-toolkit
// convrot_w4a8_quant.py, _w4a8_linear_ste_op: unpack to the int8 grid, then
// torch._int_mm and the epilogue), but the int8 weight never exists in
// global memory: each stage's weight tile is decoded from the packed codes,
// the fp8 group scales and the codebook straight into the shared-memory
// layout the tensor cores read.
//
// Per CTA pair and 256 x 256 output tile, per 128-wide K stage:
//   warp 0      TMA: this CTA's 128-row half of the A tile (to the leader's
//               stage barrier, as in gm::gemm_pair_kernel), and the packed
//               codes (128 rows x 64 B) and scale bytes of this CTA's 128-row
//               half of the B tile (to a CTA-local barrier);
//   warps 6-13  decode those 128 rows x 128 k into the B half of the stage,
//               in the 128-byte-swizzled K-major layout a TMA copy would have
//               produced (row r at r * 128 B, 16-byte chunk j at j ^ (r % 8)),
//               then fence the writes for the tensor cores and arrive on the
//               leader's stage barrier;
//   warp 1      the leader's MMA issuer: tcgen05.mma cta_group::2 kind::i8
//               (M 256, N 256, K 32) once the A bytes have landed and all 16
//               decode warps of the pair have arrived;
//   warps 2-5   the epilogue of gm::gemm_pair_kernel.
// The decode of a stage (16 K weights per CTA, byte permutes through a per-CTA
// table of the 16 int8 levels of every fp8 scale byte) overlaps the MMAs of
// the previous stages; per SM it needs about half of the ALU pipe while the
// tensor pipe is busy.
#pragma once

#include "k_gemm.cuh"

namespace cr {
namespace gd {

using gm::BK;
using gm::BN;
using gm::kEpiBytes;
using gm::kTmemCols;

constexpr int kDecodeWarps = 8;
constexpr int kFirstDecodeWarp = 6;
constexpr int kThreads = (kFirstDecodeWarp + kDecodeWarps) * 32;  // 448
constexpr int kStages = 4;
constexpr int kHalfBytes = 128 * BK;    // 16 KB: one CTA's half of A or of B (int8)
constexpr int kCodeBytes = 128 * BK / 2;  // 8 KB: packed codes of the B half
constexpr int kSrelBytes = 128 * 16;      // 2 KB: scale bytes of two K blocks per row
constexpr int kLutCopies = 8;
constexpr uint32_t kIdesc = idesc_i8(256, BN);
// leader's stage barrier: the producer's expect-tx arrival + every decode warp of both CTAs
constexpr uint32_t kFullCount = 1 + 2 * kDecodeWarps;

struct __align__(1024) Smem {
    uint8_t a[kStages][kHalfBytes];     // A half, 128-byte swizzled (TMA)
    uint8_t b[kStages][kHalfBytes];     // B half, 128-byte swizzled (decode warps)
    uint8_t codes[kStages][kCodeBytes]; // [128 rows][64 B] packed codes of the stage
    uint8_t srel[kStages][kSrelBytes];  // [128 rows][16 B] scale bytes of K blocks 2i, 2i+1
    uint4 lut[256 * kLutCopies];        // lut[s * kLutCopies + c]: copy c of the levels of scale byte s
    uint8_t epi[4][kEpiBytes];
    float wsb[2][BN];
    float biasb[2][BN];
    float cb[16];
    uint64_t full[kStages];      // leader: A bytes of both CTAs + all decode warps of the pair
    uint64_t raw_full[kStages];  // each CTA: its packed codes and scales have landed
    uint64_t empty[kStages];     // each CTA: the stage's MMAs are done
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint32_t tmem_base;
    int abort;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory of the fused GEMM");

__device__ __forceinline__ void decode_sync() { asm volatile("bar.sync 3, %0;" ::"n"(kDecodeWarps * 32) : "memory"); }

// tmA: xq as in gm::gemm_pair_kernel (box 128 rows x 128 k, 128-byte swizzle).
// tmQ: the packed codes, uint8 [N, K/2], box {64, 128 rows}, no swizzle.
// tmS: the scale bytes, uint8 [N, K/16], box {16, 128 rows}, no swizzle; a
//      stage loads the 16 bytes of K blocks 2i and 2i + 1 (x must stay a
//      multiple of 16 bytes) and uses the half of its own block.
__global__ void __launch_bounds__(kThreads, 1)
    gemm_dec_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmOut,
                         const float *__restrict__ codebook, const float *__restrict__ xs,
                         const float *__restrict__ ws, const float *__restrict__ bias, int M, int N, int K,
                         int out_f32, int tma_out, void *__restrict__ out, int32_t *__restrict__ acc_out)
{
    extern __shared__ uint8_t smem_raw[];
    Smem &sh = smem_aligned_1024<Smem>(smem_raw);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int npairs = gridDim.x >> 1, pair_id = blockIdx.x >> 1;
    const int tiles_m = (M + 255) / 256, tiles_n = (N + BN - 1) / BN;
    const int num_tiles = tiles_m * tiles_n;
    const int kblocks = K / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sh.full[s], kFullCount);
            mbar_init(&sh.raw_full[s], 1);
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
    if (threadIdx.x < 16)
        sh.cb[threadIdx.x] = codebook[threadIdx.x];
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
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmS);
            int stage = 0;
            uint32_t phase = 0;
            int issued[kStages];
            uint32_t issued_phase[kStages];
            for (int s = 0; s < kStages; ++s)
                issued[s] = 0, issued_phase[s] = 0;
            bool ok = true;
            for (int tile = pair_id; ok && tile < num_tiles; tile += npairs) {
                int tm, tn;
                gm::tile_coords(tile, tiles_n, tm, tn);
                const int brow = tn * BN + (int)rank * 128;  // this CTA's rows of the B tile
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait_bounded(&sh.empty[stage], phase ^ 1u, abort)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full_leader = mapa_shared(smem_u32(&sh.full[stage]), 0);
                    if (leader)
                        mbar_arrive_expect_tx(&sh.full[stage], 2 * kHalfBytes);
                    tma_load_2d_pair(sh.a[stage], &tmA, kb * BK, tm * 256 + (int)rank * 128, full_leader);
                    mbar_arrive_expect_tx(&sh.raw_full[stage], kCodeBytes + kSrelBytes);
                    tma_load_2d(sh.codes[stage], &tmQ, kb * (BK / 2), brow, &sh.raw_full[stage]);
                    tma_load_2d(sh.srel[stage], &tmS, (kb & ~1) * (BK / 16), brow, &sh.raw_full[stage]);
                    issued[stage] = 1;
                    issued_phase[stage] = phase;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // let copies in flight land before the CTAs go away (see gm::gemm_pair_kernel)
                for (int s = 0; s < kStages; ++s)
                    if (issued[s]) {
                        volatile int no_abort = 0;
                        mbar_wait_bounded(&sh.raw_full[s], issued_phase[s], &no_abort, 20000000ull);
                    }
                if (leader) {
                    for (int s = 0; s < kStages; ++s)
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
                    const uint32_t a_addr = smem_u32(sh.a[stage]);
                    const uint32_t b_addr = smem_u32(sh.b[stage]);
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk)
                        mma_i8_pair(d, sw128_kmajor_desc(a_addr + 32u * kk), sw128_kmajor_desc(b_addr + 32u * kk),
                                    kIdesc, (kb | kk) != 0 ? 1u : 0u);
                    const uint32_t e = smem_u32(&sh.empty[stage]);
                    tc_commit_pair(mapa_shared(e, 0));
                    tc_commit_pair(mapa_shared(e, peer));
                    if (++stage == kStages) {
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
    } else if (warp < kFirstDecodeWarp) {
        // ------------------------------------------------ epilogue (warps 2..5, both CTAs)
        const int q = warp & 3;
        const int et = threadIdx.x - 64;
        int local = 0;
        uint32_t units_issued = 0;
        for (int tile = pair_id; tile < num_tiles; tile += npairs, ++local) {
            int tm, tn;
            gm::tile_coords(tile, tiles_n, tm, tn);
            const int buf = local & 1;
            const uint32_t use = (uint32_t)(local >> 1) & 1u;
            for (int j = et; j < BN; j += 128) {
                const int n = tn * BN + j;
                sh.wsb[buf][j] = n < N ? ws[n] : 0.0f;
                sh.biasb[buf][j] = (bias != nullptr && n < N) ? bias[n] : 0.0f;
            }
            asm volatile("bar.sync 2, 128;" ::: "memory");
            const bool ok = mbar_wait_bounded_warp(&sh.tmem_full[buf], use, abort);
            if (!ok)
                continue;
            tc_fence_after();
            const int row0 = tm * 256 + (int)rank * 128 + 32 * q;
            const bool row_ok = row0 + lane < M;
            const float xm = row_ok ? xs[row0 + lane] : 0.0f;
            const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * BN);
            const uint32_t release_addr = mapa_shared(smem_u32(&sh.tmem_empty[buf]), 0);
            gm::epilogue_tile(tbase, row0, tn * BN, lane, xm, row_ok, sh.wsb[buf], sh.biasb[buf], bias != nullptr, M,
                              N, out_f32, tma_out, &tmOut, sh.epi[q], units_issued, out, acc_out, ws, bias, [&]() {
                                  tc_fence_before();
                                  __syncwarp();
                                  if (lane == 0)
                                      mbar_arrive_cluster(release_addr);
                              });
        }
        if (lane == 0)
            bulk_wait_all();
        __syncwarp();
    } else {
        // ------------------------------------------------ decode warps (both CTAs)
        const int dt = threadIdx.x - kFirstDecodeWarp * 32;  // 0 .. 255
        {
            const uint4 e = lut_entry((uint32_t)dt, sh.cb);
#pragma unroll
            for (int r = 0; r < kLutCopies; ++r)
                sh.lut[dt * kLutCopies + ((r + dt) & (kLutCopies - 1))] = e;
        }
        decode_sync();
        // Each warp decodes 16 rows of the B half per stage: per pass, lane
        // (row r0 + lane / 8, 16-column chunk j = lane % 8), four passes.
        const int dw = warp - kFirstDecodeWarp;
        const int j = lane & 7;
        const uint4 *lutc = sh.lut + (lane & (kLutCopies - 1));
        int stage = 0;
        uint32_t phase = 0;
        for (int tile = pair_id; tile < num_tiles; tile += npairs) {
            for (int kb = 0; kb < kblocks; ++kb) {
                const bool ok = mbar_wait_bounded_warp(&sh.raw_full[stage], phase, abort);
                if (ok) {
                    const uint8_t *codes = sh.codes[stage];
                    const uint8_t *srel = sh.srel[stage] + (kb & 1) * 8 + j;
                    uint8_t *b = sh.b[stage];
#pragma unroll
                    for (int pass = 0; pass < 4; ++pass) {
                        const int r = dw * 16 + pass * 4 + (lane >> 3);
                        const uint2 c = *reinterpret_cast<const uint2 *>(codes + r * (BK / 2) + j * 8);
                        const uint4 T = lutc[kLutCopies * (uint32_t)srel[r * 16]];
                        uint4 w;
                        decode8(c.x, T, w.x, w.y);
                        decode8(c.y, T, w.z, w.w);
                        *reinterpret_cast<uint4 *>(b + r * 128 + ((j ^ (r & 7)) << 4)) = w;
                    }
                    // the tensor cores read this stage through the async proxy
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                }
                __syncwarp();
                if (ok && lane == 0)
                    mbar_arrive_remote(mapa_shared(smem_u32(&sh.full[stage]), 0));
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // no CTA leaves while its partner may still signal it
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

}  // namespace gd
}  // namespace cr
