// k_peak.cuh -- measurement kernel: the dense INT8 tensor-core rate of this
// GPU, for the prefill GEMM's roofline.
//
// Every SM pair (cluster of two CTAs) keeps one 256 x 128 int8 A tile and one
// 256 x 128 int8 B tile resident in shared memory (each CTA holds its 128-row
// halves, filled with pseudo-random bytes) and issues `iters` groups of four
// tcgen05.mma.cta_group::2.kind::i8 (M = 256, N = 256, K = 32) into one TMEM
// accumulator, exactly the instruction shape and operand layout of the
// prefill GEMM's CTA-pair kernel, with no memory traffic.  A final commit
// signals both CTAs; the host times the launch with CUDA events.  Ops per
// launch: 2 * 256 * 256 * 128 * iters per pair.
#pragma once

#include "cr_device.cuh"

namespace cr {
namespace pk {

constexpr int kThreads = 128;
constexpr int kHalfBytes = 128 * 128;  // one CTA's 128 rows x 128 bytes of A (and of B)

struct __align__(1024) Smem {
    uint8_t a[kHalfBytes];
    uint8_t b[kHalfBytes];
    uint64_t done;
    uint32_t tmem_base;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

__global__ void __launch_bounds__(kThreads, 1) mma_i8_peak_kernel(int iters)
{
    extern __shared__ uint8_t smem_raw[];
    Smem &sh = smem_aligned_1024<Smem>(smem_raw);
    const int warp = threadIdx.x >> 5;
    const uint32_t rank = cluster_ctarank();

    // operands: a xorshift stream of bytes per thread (values do not matter
    // for the rate, but random bits draw the power real data draws)
    uint32_t st = 0x9E3779B9u * (threadIdx.x + 1) + 0x85EBCA6Bu * (blockIdx.x + 1);
    for (int i = threadIdx.x * 4; i < 2 * kHalfBytes; i += kThreads * 4) {
        st ^= st << 13;
        st ^= st >> 17;
        st ^= st << 5;
        *reinterpret_cast<uint32_t *>(sh.a + i) = st;  // a and b are contiguous
    }
    fence_async_smem();
    if (threadIdx.x == 0) {
        mbar_init(&sh.done, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        tmem_alloc_pair(&sh.tmem_base, 256);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    volatile int abort = 0;

    if (rank == 0 && threadIdx.x == 0) {
        const uint32_t a_addr = smem_u32(sh.a), b_addr = smem_u32(sh.b);
        constexpr uint32_t idesc = idesc_i8(256, 256);
        for (int it = 0; it < iters; ++it) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_i8_pair(tmem, sw128_kmajor_desc(a_addr + 32u * kk), sw128_kmajor_desc(b_addr + 32u * kk), idesc,
                            (it | kk) != 0 ? 1u : 0u);
        }
        const uint32_t d = smem_u32(&sh.done);
        tc_commit_pair(mapa_shared(d, 0));
        tc_commit_pair(mapa_shared(d, 1));
    }
    if (threadIdx.x == 0)
        mbar_wait_bounded(&sh.done, 0, &abort);
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, 256);
    }
}

}  // namespace pk
}  // namespace cr
