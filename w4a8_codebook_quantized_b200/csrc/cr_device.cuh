// cr_device.cuh -- device helpers shared by the sm_100a kernels of the ConvRot
// W4A8 codebook linear layer: fp8 scale decode, the per-CTA int8-grid lookup
// table, nibble decode by byte permutes, the epilogue, the library error word,
// and thin PTX wrappers for mbarriers, TMA, tcgen05 and TMEM.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "cr_w4a8.h"

namespace cr {

// Set by a kernel whose bounded pipeline wait ran out; read and cleared by
// cr_check_device_error().  One per device (module-scope __device__ variable;
// the library is a single translation unit, so it is defined here).
__device__ int g_device_error = 0;

enum : int { kErrTimeout = 1 };

// ---------------------------------------------------------------- fp8 scales

// fp8 e4m3fn byte -> fp32, exact.  Format (ai-toolkit convrot_w4a8_quant.py,
// w4a8_gemv_kernel: the s_rel byte is read as float8e4nv): sign, 4 exponent
// bits with bias 7, 3 mantissa bits, no infinities, S.1111.111 is NaN.
// Normal values are rebuilt as fp32 bit fields (exponent e - 7 + 127 = e + 120,
// mantissa in the top three fraction bits); subnormals are m * 2^-9.
__device__ __forceinline__ float fp8e4m3fn_to_float(uint32_t b)
{
    const uint32_t sign = (b & 0x80u) << 24;
    const uint32_t e = (b >> 3) & 0xFu;
    const uint32_t m = b & 0x7u;
    if (e == 0xFu && m == 0x7u)
        return __uint_as_float(0x7FC00000u | sign);
    float mag = (e == 0u) ? __fmul_rn((float)m, 0.001953125f)
                          : __uint_as_float(((e + 120u) << 23) | (m << 20));
    return __uint_as_float(__float_as_uint(mag) | sign);
}

// Round to nearest even and saturate to [-128, 127] in one conversion; NaN -> 0
// (ai-toolkit convrot_w4a8_quant.py, _sat_s8 / W4A8_SAT).
__device__ __forceinline__ int32_t sat_s8_rne(float v)
{
    int32_t r;
    asm("cvt.rni.sat.s8.f32 %0, %1;" : "=r"(r) : "f"(v));
    return r;
}

// ---------------------------------------------------------------- int8-grid LUT
//
// The decoded weight depends only on (scale byte, code): w8 = sat_s8(rne(cb[code]
// * fp8(s))).  A CTA tabulates all 256 x 16 values once; entry s is one uint4
// whose 16 bytes are the levels of codes 0..15 (x: codes 0-3, y: 4-7, z: 8-11,
// w: 12-15).
__device__ __forceinline__ uint4 lut_entry(uint32_t s, const float *cb /* 16, any memory */)
{
    const float sv = fp8e4m3fn_to_float(s);
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int32_t l = sat_s8_rne(__fmul_rn(cb[4 * q + j], sv));
            word |= ((uint32_t)l & 0xFFu) << (8 * j);
        }
        w[q] = word;
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// The split form of a level table (the fast decode of the decode GEMV): from
// the 16 levels L of `e` (lut_entry), two 8-byte tables P (x, y) and Q (z, w)
// with, for each j = 0..7, P[j] + sgn(Q[j]) = L[j] and sgn(P[j]) + Q[j] =
// L[j + 8], where sgn(v) is -1 for a negative byte and 0 otherwise (what a
// sign-replicating byte permute returns).  Taking P[j] = L[j] + a and
// Q[j] = L[j + 8] + b with a = [Q[j] < 0], b = [P[j] < 0] always has an int8
// solution unless one of the two levels is 127 and the other negative; ok is
// cleared for such a table.
__device__ __forceinline__ uint4 lut_entry_split(const uint4 &e, bool &ok)
{
    const uint32_t w[4] = {e.x, e.y, e.z, e.w};
    uint32_t P[2] = {0u, 0u}, Q[2] = {0u, 0u};
    ok = true;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int p = (int)(int8_t)(w[j >> 2] >> (8 * (j & 3)));
        const int q = (int)(int8_t)(w[2 + (j >> 2)] >> (8 * (j & 3)));
        int A = p, B = q + (p < 0 ? 1 : 0);  // a = 0: needs Q[j] = B >= 0
        if (B < 0 || B > 127) {
            A = p + 1;                        // a = 1: needs Q[j] < 0
            B = q + (A < 0 ? 1 : 0);
            if (p > 126 || B >= 0) {
                ok = false;
                A = 0;
                B = 0;
            }
        }
        P[j >> 2] |= ((uint32_t)A & 0xFFu) << (8 * (j & 3));
        Q[j >> 2] |= ((uint32_t)B & 0xFFu) << (8 * (j & 3));
    }
    return make_uint4(P[0], P[1], Q[0], Q[1]);
}

// PTX prmt in its default mode: selector nibble i = {sign-replicate bit, 3-bit
// source byte index} for output byte i; source bytes 0-3 from a, 4-7 from b.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Decode 8 packed codes (one 32-bit word: nibble i = code of column base + i,
// which is the storage order: even column in the low nibble) through the level
// table T of their group.  Returns the int8 grid values of columns 0-3 in w0
// and 4-7 in w1 (byte i of w0 = column i).
//
// Byte permutes do the table lookup: the low three bits of each code select
// among levels 0-7 (T.x:T.y) and among levels 8-15 (T.z:T.w); bit 3 picks one
// of the two.  The bit-3 byte mask comes from prmt's sign-replicate mode
// applied to the code word and the code word shifted left by 4, whose bytes
// carry code bit 3 in their sign bit.
__device__ __forceinline__ void decode8(uint32_t c, const uint4 &T, uint32_t &w0, uint32_t &w1)
{
    const uint32_t s7 = c & 0x77777777u;
    const uint32_t s7h = s7 >> 16;
    const uint32_t lo0 = prmt(T.x, T.y, s7);
    const uint32_t hi0 = prmt(T.z, T.w, s7);
    const uint32_t lo1 = prmt(T.x, T.y, s7h);
    const uint32_t hi1 = prmt(T.z, T.w, s7h);
    const uint32_t c4 = c << 4;
    // output byte i <- sign of: (c4 byte 0), (c byte 0), (c4 byte 1), (c byte 1)
    const uint32_t m0 = prmt(c4, c, 0xD9C8u);
    // ... and for codes 4-7: (c4 byte 2), (c byte 2), (c4 byte 3), (c byte 3)
    const uint32_t m1 = prmt(c4, c, 0xFBEAu);
    w0 = (hi0 & m0) | (lo0 & ~m0);
    w1 = (hi1 & m1) | (lo1 & ~m1);
}

// ---------------------------------------------------------------- epilogue
//
// ai-toolkit convrot_w4a8_quant.py, w4a8_gemv_kernel epilogue:
// float(acc) * (xs * ws) [+ bias], each operation rounded on its own.
__device__ __forceinline__ float epilogue_value(int32_t acc, float xs, float ws, const float *bias,
                                                int64_t n)
{
    float y = __fmul_rn(__int2float_rn(acc), __fmul_rn(xs, ws));
    if (bias != nullptr)
        y = __fadd_rn(y, bias[n]);
    return y;
}

// SwiGLU of one gate/up pair of epilogue values (h3-rs weights.rs,
// swiglu_interleaved): silu(g) * u = g * sigmoid(g) * u, in fp32.  With
// t = e^-|g| (CUDA's expf; t lies in (0, 1], so it never overflows):
//   silu(g) = g / (1 + t)        for g >= 0
//           = g * t / (1 + t)    for g <  0   (the same value, e^g = t)
// so the divisor always lies in [1, 2], where the fast division __fdividef
// has at most 2 ulp of error (outside [2^-126, 2^126] it does not: a divisor
// 1 + e^-g near 2^127 would return 0 for gates around -88, and e^-g overflows
// below -88.7, where the true result is still a normal fp32 number).  The
// IEEE division's slow-path branch would keep the compiler from overlapping
// the independent pairs of a thread; this form has no branch.
__device__ __forceinline__ float swiglu_value(float g, float u)
{
    const float t = expf(-fabsf(g));
    const float num = g >= 0.0f ? g : __fmul_rn(g, t);
    return __fmul_rn(__fdividef(num, __fadd_rn(1.0f, t)), u);
}

__device__ __forceinline__ uint16_t to_bf16_bits(float y)
{
    return __bfloat16_as_ushort(__float2bfloat16_rn(y));
}

// Two values to a pair of bf16 (round to nearest even) in one conversion:
// lo in bits 0-15, hi in bits 16-31.
__device__ __forceinline__ uint32_t to_bf16x2_bits(float lo, float hi)
{
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&p);
}

// ---------------------------------------------------------------- loads

// 8-byte streaming load that bypasses L1 (weights are read once).
__device__ __forceinline__ uint2 ldg_stream8(const void *p)
{
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Arrive without release ordering.  For a consumer handing a ring stage back
// after every value it read from the stage has been used in registers: no
// ordering of its other (global) memory operations is needed, and a release
// arrive would wait for this thread's outstanding prefetch loads.
__device__ __forceinline__ void mbar_arrive_relaxed(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait for the phase with the given parity to complete.  Gives up
// after `limit_ns` of wall time, or as soon as *abort is set by another warp
// of the CTA; on giving up it sets *abort and the device error word and
// returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort,
                                                  uint64_t limit_ns = 2000000000ull)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((it & 63u) == 0u) {
            if (*abort)
                return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                *abort = 1;
                atomicExch(&g_device_error, kErrTimeout);
                return false;
            }
        }
    }
}

// The same bounded wait, taken by a whole warp: every lane polls, and the
// outcome is the same in all lanes (warp-collective instructions follow it).
__device__ __forceinline__ bool mbar_wait_bounded_warp(uint64_t *bar, uint32_t parity, volatile int *abort,
                                                       uint64_t limit_ns = 2000000000ull)
{
    if (__all_sync(0xFFFFFFFFu, mbar_try_wait(bar, parity)))
        return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (__all_sync(0xFFFFFFFFu, mbar_try_wait(bar, parity)))
            return true;
        if ((it & 63u) == 0u) {
            int give_up = 0;
            if ((threadIdx.x & 31) == 0) {
                if (*abort) {
                    give_up = 1;
                } else if (globaltimer_ns() - t0 > limit_ns) {
                    *abort = 1;
                    atomicExch(&g_device_error, kErrTimeout);
                    give_up = 1;
                }
            }
            if (__shfl_sync(0xFFFFFFFFu, give_up, 0))
                return false;
        }
    }
}

// ---------------------------------------------------------------- TMA

// The dynamic shared-memory buffer rounded up to a 1024-byte boundary (the
// alignment the 128-byte-swizzled TMA layouts need).  The padding is added to
// the __shared__ array itself rather than to an integer copy of its address,
// so the result stays in the shared state space and its reads compile to
// shared-memory loads instead of generic ones.
template <class T>
__device__ __forceinline__ T &smem_aligned_1024(uint8_t *smem_raw)
{
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    return *reinterpret_cast<T *>(smem_raw + pad);
}

// Prefetch of a 3-D tile into L2 (no shared memory, no completion to track;
// out-of-range parts of the box are ignored).
__device__ __forceinline__ void tma_prefetch_3d(const void *tmap, int32_t x, int32_t y, int32_t z)
{
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(tmap), "r"(x), "r"(y),
                 "r"(z)
                 : "memory");
}

// 3-D tiled bulk tensor load into this CTA's shared memory.
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const void *tmap, int32_t x, int32_t y, int32_t z,
                                            uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
            smem_u32(smem_dst)),
        "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_2d(void *smem_dst, const void *tmap, int32_t x, int32_t y, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(smem_dst)),
        "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Bring [p, p + bytes) into L2 (16-byte aligned address, size a multiple of
// 16).  A hint with no effect on the values any load returns.
__device__ __forceinline__ void bulk_prefetch_l2(const void *p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void *tmap)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// Bulk tensor store of one box from shared memory (shared::cta source), in
// the calling thread's bulk-async group.  Out-of-range parts of the box are
// not written.
__device__ __forceinline__ void tma_store_2d(const void *tmap, int32_t x, int32_t y, const void *smem_src)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(tmap), "r"(x),
                 "r"(y), "r"(smem_u32(smem_src))
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N committed bulk groups still read their shared-memory source.
template <int N>
__device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until every committed bulk group has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (TMA) before a bulk copy reads them.
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---------------------------------------------------------------- tcgen05 / TMEM

__device__ __forceinline__ void tmem_alloc(uint32_t *smem_result, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_result)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive on an mbarrier once every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void tc_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// D[tmem] (+)= A[smem] x B[smem]^T, int8 x int8 -> int32.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[smem] x B[smem]^T, bf16 x bf16 -> fp32 (kind::f16; A and B
// of the same type).
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 consecutive 32-bit TMEM columns of this warp's 32 lanes -> 32 registers.
__device__ __forceinline__ void tmem_ld_32cols(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait()
{
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- CTA pairs (cluster of 2)

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// The shared::cluster address of the same shared-memory location in CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t smem_addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}

// All threads of both CTAs of the pair.
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on an mbarrier given by a shared::cluster address (this CTA's or the peer's).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// TMA tile load into this CTA's shared memory whose completion is signalled on
// an mbarrier that may live in either CTA of the pair (shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void *smem_dst, const void *tmap, int32_t x, int32_t y,
                                                 uint32_t mbar_cluster_addr)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(smem_dst)),
        "l"(tmap), "r"(x), "r"(y), "r"(mbar_cluster_addr)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t *smem_result, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_result)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Arrive on the mbarrier at `cluster_addr` once every tcgen05 operation this
// thread issued for the pair has completed.
__device__ __forceinline__ void tc_commit_pair(uint32_t cluster_addr)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(cluster_addr)
                 : "memory");
}

// D[tmem] (+)= A x B^T over the CTA pair: M = 256 (128 rows of A from each
// CTA's shared memory at the descriptor's offset), B split the same way.
__device__ __forceinline__ void mma_i8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The same over the CTA pair for kind::f16 (bf16 x bf16 -> fp32).
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile stored in the
// 128-byte-swizzled canonical layout: rows of 128 bytes, 8-row atoms of 1024
// bytes stacked along the row dimension (stride-dimension byte offset 1024).
// Fields: start address >> 4 in bits 0-13, leading byte offset >> 4 in 16-29
// (unused for swizzled K-major tiles; set to 1), stride byte offset >> 4 in
// 32-45, descriptor version 1 in bits 46-47, swizzle mode 2 (128 B) in 61-63.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr)
{
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// Instruction descriptor for kind::i8: s32 accumulator, signed A and B, both
// K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N)
{
    return (2u << 4)                        // D format: s32
           | (1u << 7)                      // A: signed 8-bit
           | (1u << 10)                     // B: signed 8-bit
           | ((uint32_t)(N >> 3) << 17)     // N / 8
           | ((uint32_t)(M >> 4) << 24);    // M / 16
}

// Instruction descriptor for kind::f16 with bf16 A and B and an fp32
// accumulator, both operands K-major: D format 1 (f32) in bits 4-5, A and B
// format 1 (bf16) in bits 7-9 and 10-12, N / 8 in bits 17-22, M / 16 in 24-28.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N)
{
    return (1u << 4)                        // D format: f32
           | (1u << 7)                      // A: bf16
           | (1u << 10)                     // B: bf16
           | ((uint32_t)(N >> 3) << 17)     // N / 8
           | ((uint32_t)(M >> 4) << 24);    // M / 16
}

}  // namespace cr
