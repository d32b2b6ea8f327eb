// k_gemv.cuh -- fused decode GEMV for M <= 8 tokens.
//
// What it computes (ai-toolkit convrot_w4a8_quant.py, w4a8_gemv_kernel):
// out[m, n] = epilogue(sum_k xq[m, k] * w8[n, k]) with w8 decoded on the fly
// from the packed codes, the fp8 group scales and the codebook, so the weight
// costs 4.5 bits of HBM traffic and is never materialised.  The int32 sums
// are exact, so the result equals the prefill path bit for bit.
//
// B200 design.
//  * Streaming: a persistent grid (two CTAs per SM).  In each CTA one
//    producer warp moves, per stage, the packed codes of a row tile (16 or
//    32 weight rows x 1024 columns, 8 or 16 KB), their group scales (1 or
//    2 KB) and the matching 1024 columns of the M <= 8 activation rows (M KB)
//    into a ring of shared-memory stages with 3-D TMA copies; eight consumer warps decode and contract each
//    stage while the following ones are in flight; an epilogue warp reduces
//    the consumers' partial sums and writes the outputs of a tile while the
//    consumers already work on the next one.  Bytes in flight are set by the
//    ring, not by registers, and the consumers issue no global memory
//    accesses and take no CTA-wide barrier in the loop.
//  * Shared-memory layouts chosen for conflict-free reads: the tensor maps
//    order the box so that a stage holds the codes as [slice][row][64 B], the
//    scales as [256-column block][row][16 B] and the activations as
//    [slice][token < M][128 B] with the 128-byte swizzle; every quarter-warp
//    request then touches 8 distinct 16-byte bank groups.  The activation box
//    has exactly M rows: no rows are zero-filled by the copy engine (which
//    measurably slows a stage), and the stage carries M KB of activations
//    rather than 8.  Lanes of tokens m >= M read stale bytes of the stage;
//    they only feed accumulator columns that are never written out.
//  * Decode: a per-CTA table of the 16 int8 levels of every fp8 scale byte
//    (exact: the decoded value depends only on the pair), replicated so that
//    the lanes of a quarter-warp mostly read distinct bank groups; byte
//    permutes turn 8 packed codes into 8 int8 levels.
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
//  * Tile height: with 32-row tiles a stage's activation copy and each
//    thread's activation fragments serve two MMA row blocks (rows 0-15 and
//    16-31), which halves the activation traffic into shared memory and the
//    per-stage ring overhead per weight.  Measured on B200, a stage's
//    activation copy costs far more than its bytes (removing it entirely took
//    an M = 8, N = K = 8192 GEMV from 11.1 to 9.3 us; spreading its reads over
//    16 copies in L2 changed nothing), so the copies per weight are what
//    matters.  Layers with fewer tiles than SMs keep 16-row tiles, which
//    spread them over more SMs.
//  * Launch overlap: the kernel lets the next kernel on the stream launch at
//    once, and it may itself start before the previous kernel ends (weight
//    stream and table build first); the activation copies and every read of
//    xq / xs and write of the outputs wait for that kernel
//    (griddepcontrol.wait).
#pragma once

#include <cuda.h>

#include "cr_device.cuh"

namespace cr {
namespace gv {

constexpr int kConsumerWarps = 8;
constexpr int kProducerWarp = kConsumerWarps;       // TMA issue
constexpr int kEpilogueWarp = kConsumerWarps + 1;   // reduction, split-tile hand-off, outputs
constexpr int kThreads = (kConsumerWarps + 2) * 32;
constexpr int kMmaRows = 16;                         // weight rows of one MMA (its M)
constexpr int kSlice = 128;                          // columns per consumer warp per stage
constexpr int kChunk = kConsumerWarps * kSlice;      // columns per stage
constexpr int kTokens = 8;                           // activation rows of a stage (the MMA's N)
constexpr int kXBytes = kTokens * kChunk;  // room for M = 8; a stage carries M * kChunk
// L2 prefetch distance of the weight stream beyond the ring, in stages.
// Measured on B200 with the current rings (A/B in both build orders): 0 beats
// 3 on the large layers (M = 8, N = K = 8192: 11.0 -> 10.5 us; 16384^2:
// 37.7 -> 34.6 us) and ties elsewhere, so the prefetch is off; the mechanism
// stays for other ring depths.
constexpr int kPrefetchAhead = 0;
constexpr int kRedBufs = 1;  // partial-sum mailboxes between the consumers and the epilogue warp

// Shape of the ring: STAGES stages, MINB CTAs per SM, COPIES copies of the
// level table (8 copies make every quarter-warp lookup conflict-free, 4 leave
// occasional two-way conflicts for half the shared memory), ROWS weight rows
// per tile: 16 (one MMA row block), or 32 (two row blocks that share every
// activation stage and every activation fragment, so that a stage's
// activation copy serves twice the weights).
template <int STAGES, int MINB, int COPIES, int ROWS>
struct Cfg {
    static constexpr int kStages = STAGES;
    static constexpr int kMinBlocks = MINB;
    static constexpr int kCopies = COPIES;
    static constexpr int kRows = ROWS;
    static constexpr int kBlocks = ROWS / kMmaRows;  // MMA row blocks per tile
    static constexpr int kCodeBytes = ROWS * kChunk / 2;
    static constexpr int kSrelBytes = ROWS * kChunk / 16;
    struct __align__(1024) Smem {
        uint8_t x[STAGES][kXBytes];          // [slice][token < M][128 B], 128-byte swizzle (1024-aligned)
        uint8_t codes[STAGES][kCodeBytes];   // [slice][row][64 B]
        uint8_t srel[STAGES][kSrelBytes];    // [256-column block][row][16 B]
        uint4 lut[256 * COPIES];             // lut[s * COPIES + c]: copy c of the levels of scale byte s
        int32_t red[kRedBufs][kConsumerWarps][ROWS][8];  // per-warp partial sums
        alignas(16) uint16_t ostage[kTokens][ROWS];      // a tile's bf16 outputs, token-major
        float cb[16];
        uint64_t full[STAGES];
        uint64_t empty[STAGES];
        uint64_t red_full[kRedBufs];   // the eight consumer warps have written red[b]
        uint64_t red_empty[kRedBufs];  // the epilogue warp has read red[b]
        int abort;
    };
    static constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
};

// The configurations the library launches: 16-row tiles, and 32-row tiles
// for single layers with enough rows to fill the SMs with them.
using Prod = Cfg<5, 2, 4, 16>;
using Prod32 = Cfg<3, 2, 4, 32>;

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

// The operands of one stage for one thread and one MMA row block: the
// activation fragments (shared by the tile's row blocks), the 32 codes of
// rows g and g + 8, and the level tables of their two groups.
struct Ops {
    uint4 X0, X1, A, B, TA0, TA1, TB0, TB1;
};

// Fetch a stage's operands from shared memory.  `lutb` points at this lane's
// copy of the level table; the entry of scale byte s sits s * lut_step bytes
// further.  lut_step is a kernel argument rather than a constant so that the
// address is one integer multiply-add, which issues on the FMA pipe and leaves
// the ALU pipe, the decode's bottleneck, to the byte permutes.
__device__ __forceinline__ void fetch_w(Ops &o, const uint8_t *codes_g, const uint8_t *srel_g, const uint8_t *lutb,
                                        uint32_t lut_step)
{
    o.A = *reinterpret_cast<const uint4 *>(codes_g);
    o.B = *reinterpret_cast<const uint4 *>(codes_g + 8 * 64);
    o.TA0 = *reinterpret_cast<const uint4 *>(lutb + (uint32_t)srel_g[0] * lut_step);
    o.TA1 = *reinterpret_cast<const uint4 *>(lutb + (uint32_t)srel_g[1] * lut_step);
    o.TB0 = *reinterpret_cast<const uint4 *>(lutb + (uint32_t)srel_g[8 * 16] * lut_step);
    o.TB1 = *reinterpret_cast<const uint4 *>(lutb + (uint32_t)srel_g[8 * 16 + 1] * lut_step);
}

// One slice of the tile: rows g and g + 8 x 128 k against the token
// fragments, into the two accumulators.
__device__ __forceinline__ void slice_mma(const Ops &o, int32_t (&c)[4], int32_t (&d)[4])
{
    uint32_t a0, a1, a2, a3, e0, e1, e2, e3;
    decode8(o.A.x, o.TA0, a0, a2);
    decode8(o.B.x, o.TB0, a1, a3);
    decode8(o.A.y, o.TA0, e0, e2);
    decode8(o.B.y, o.TB0, e1, e3);
    mma_s8(c, a0, a1, a2, a3, o.X0.x, o.X0.y);
    mma_s8(d, e0, e1, e2, e3, o.X0.z, o.X0.w);
    decode8(o.A.z, o.TA1, a0, a2);
    decode8(o.B.z, o.TB1, a1, a3);
    decode8(o.A.w, o.TA1, e0, e2);
    decode8(o.B.w, o.TB1, e1, e3);
    mma_s8(c, a0, a1, a2, a3, o.X1.x, o.X1.y);
    mma_s8(d, e0, e1, e2, e3, o.X1.z, o.X1.w);
}

// Split decode.  The table entry of a scale byte may hold, instead of the 16
// levels, two 8-byte tables P = T.x:T.y and Q = T.z:T.w (lut_entry_split)
// built so that, for every code c,
//   P-permute(c) + Q-permute(c ^ 8) = level(c)
// where a byte permute with selector nibble c returns table byte c for c < 8
// and, for c >= 8, the sign of table byte c - 8 replicated (0 or -1).  The two
// permute results are two int8 weights whose sum is the decoded weight, and
// the tensor core adds them: one MMA on each, with the same activations, into
// the same accumulator (exact integer sums).  Per 8 codes that is 4 permutes,
// one xor and two shifts against the 11 ALU operations of decode8, for one
// more MMA per code word.  A launch uses it (the kernel's SPLIT variant) when
// every table the layer reads has a split form, which the host establishes
// once per prepared layer (split_check_kernel), and where a CTA has at most
// two row tiles (there it was measured faster; with more tiles per CTA the
// extra MMAs cost more than the decode saves).
__device__ __forceinline__ void decode8_split(uint32_t c, const uint4 &T, uint32_t &p0, uint32_t &p1, uint32_t &q0,
                                              uint32_t &q1)
{
    const uint32_t cx = c ^ 0x88888888u;
    p0 = prmt(T.x, T.y, c);
    q0 = prmt(T.z, T.w, cx);
    p1 = prmt(T.x, T.y, c >> 16);
    q1 = prmt(T.z, T.w, cx >> 16);
}

// slice_mma on split tables.
__device__ __forceinline__ void slice_mma_split(const Ops &o, int32_t (&c)[4], int32_t (&d)[4])
{
    uint32_t pa0, pa2, qa0, qa2, pb1, pb3, qb1, qb3, ra0, ra2, sa0, sa2, rb1, rb3, sb1, sb3;
    decode8_split(o.A.x, o.TA0, pa0, pa2, qa0, qa2);
    decode8_split(o.B.x, o.TB0, pb1, pb3, qb1, qb3);
    decode8_split(o.A.y, o.TA0, ra0, ra2, sa0, sa2);
    decode8_split(o.B.y, o.TB0, rb1, rb3, sb1, sb3);
    mma_s8(c, pa0, pb1, pa2, pb3, o.X0.x, o.X0.y);
    mma_s8(d, ra0, rb1, ra2, rb3, o.X0.z, o.X0.w);
    mma_s8(c, qa0, qb1, qa2, qb3, o.X0.x, o.X0.y);
    mma_s8(d, sa0, sb1, sa2, sb3, o.X0.z, o.X0.w);
    decode8_split(o.A.z, o.TA1, pa0, pa2, qa0, qa2);
    decode8_split(o.B.z, o.TB1, pb1, pb3, qb1, qb3);
    decode8_split(o.A.w, o.TA1, ra0, ra2, sa0, sa2);
    decode8_split(o.B.w, o.TB1, rb1, rb3, sb1, sb3);
    mma_s8(c, pa0, pb1, pa2, pb3, o.X1.x, o.X1.y);
    mma_s8(d, ra0, rb1, ra2, rb3, o.X1.z, o.X1.w);
    mma_s8(c, qa0, qb1, qa2, qb3, o.X1.x, o.X1.y);
    mma_s8(d, sa0, sb1, sa2, sb3, o.X1.z, o.X1.w);
}

// The layers one launch covers: every layer is contracted with the same
// activations (xq, xs) and was quantised with the same codebook; their row
// tiles are numbered one after the other (layer l owns the tiles
// [tile0, tile0 + ceil(N / 16))).
constexpr int kMaxLayers = 4;

struct GemvLayer {
    const float *ws;    // [N] per-channel scales
    const float *bias;  // [N] or null
    void *out;          // [M, N] bf16 or fp32
    int32_t *acc_out;   // [M, N] or null
    int N;
    int tile0;
    int swiglu;         // rows interleaved as gate/up pairs; out is [M, N / 2] of silu(gate) * up
};

// tm_codes[l]: layer l's packed codes as 32-bit words, dims {16, N, K / 128},
//              strides {K / 2, 64} bytes, box {16, 16, 8}.
// tm_srel[l]:  its scale bytes, dims {16, N, K / 256}, strides {K / 16, 16}, box {16, 16, 4}.
// tm_x:        xq, dims {128, M, K / 128}, strides {K, 128}, box {128, M, 8}, 128-byte swizzle.
// lut_step:    bytes between the table entries of consecutive scale bytes in one
//              copy (kCopies * 16).  ahead: L2 prefetch distance in stages.
// L: the layer slots of the launch (1, or kMaxLayers for a grouped call), so
// a single layer keeps a small parameter block and a constant layer index.
template <int L>
struct GemvArgs {
    CUtensorMap tm_codes[L];
    CUtensorMap tm_srel[L];
    CUtensorMap tm_x;
    GemvLayer layer[L];
    const float *xs;
    const float *codebook;
    int M, K, num_layers, num_tiles, out_f32;
    uint32_t lut_step;
    int ahead;
    int tile_rows;  // the configuration's row tile height (16 or 32), for the host's launch
};

// The layer that owns global row tile `tile`.
template <int L>
__device__ __forceinline__ int layer_of(const GemvArgs<L> &a, int tile)
{
    int l = 0;
#pragma unroll
    for (int i = 1; i < L; ++i)
        if (i < a.num_layers && tile >= a.layer[i].tile0)
            l = i;
    return l;
}

// Layer and first row of global row tile `tile` (compile-time for one layer).
template <int ROWS, int L>
__device__ __forceinline__ void locate(const GemvArgs<L> &a, int tile, int &l, int &row)
{
    if constexpr (L == 1) {
        l = 0;
        row = tile * ROWS;
    } else {
        l = layer_of(a, tile);
        row = (tile - a.layer[l].tile0) * ROWS;
    }
}

// SPLIT: the level tables in split form (slice_mma_split); only for layers
// whose every scale byte has one (split_check_kernel).
template <class C, int L, bool SPLIT>
__global__ void __launch_bounds__(kThreads, C::kMinBlocks) gemv_kernel(const __grid_constant__ GemvArgs<L> a)
{
    constexpr int STAGES = C::kStages;
    using Smem = typename C::Smem;
    extern __shared__ uint8_t smem_raw[];
    Smem &sh = smem_aligned_1024<Smem>(smem_raw);
    const int M = a.M, K = a.K;
    constexpr int kRows = C::kRows, kBlocks = C::kBlocks;
    const uint32_t stage_tx = (uint32_t)(C::kCodeBytes + C::kSrelBytes + M * kChunk);

    // The next kernel on the stream may launch now: a GEMV of the next layer
    // starts its weight stream in the SM slots this grid frees, and whatever
    // it is waits (griddepcontrol.wait) for this grid before it reads any
    // result or rewrites any input of it.
    asm volatile("griddepcontrol.launch_dependents;" :::);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ntiles = a.num_tiles;
    const int nchunks = (K + kChunk - 1) / kChunk;
    // Persistent grid: this CTA takes row tiles blockIdx.x, + gridDim.x, ...,
    // each as nchunks stages; `total` stages in all.
    const int my_tiles = (int)blockIdx.x < ntiles ? (ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int total = my_tiles * nchunks;

    // The producer initialises the barriers and starts the weight stream at
    // once; the other warps pass named barrier 2 only after the
    // initialisation, and the consumers' codebook load stays off the path to
    // the first copy.
    volatile int *abort = &sh.abort;
    if (warp == kProducerWarp) {
        // ------------------------------------------------ producer
        if (lane == 0) {
            for (int s = 0; s < STAGES; ++s) {
                mbar_init(&sh.full[s], 1);
                mbar_init(&sh.empty[s], kConsumerWarps);
            }
            for (int b = 0; b < kRedBufs; ++b) {
                mbar_init(&sh.red_full[b], kConsumerWarps);
                mbar_init(&sh.red_empty[b], 1);
            }
            sh.abort = 0;
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        __syncwarp();
        asm volatile("bar.arrive 2, %0;" ::"n"(kThreads) : "memory");
        if (lane == 0) {
            if constexpr (L == 1) {
                prefetch_tmap(&a.tm_codes[0]);
                prefetch_tmap(&a.tm_srel[0]);
            } else {
                for (int l = 0; l < a.num_layers; ++l) {
                    if (a.layer[l].N == 0)
                        continue; // its maps are left empty
                    prefetch_tmap(&a.tm_codes[l]);
                    prefetch_tmap(&a.tm_srel[l]);
                }
            }
            prefetch_tmap(&a.tm_x);
            // Stage q of this CTA's run is chunk q mod nchunks of its tile
            // q / nchunks; the producer walks these positions with counters
            // (no run-time division on its per-stage path).
            struct Pos {
                int c, tile;
            };
            auto step = [&](Pos &p) {
                if (++p.c == nchunks) {
                    p.c = 0;
                    p.tile += (int)gridDim.x;
                }
            };
            auto weights = [&](const Pos &p, int s) {
                int l, row;
                locate<C::kRows>(a, p.tile, l, row);
                tma_load_3d(sh.codes[s], &a.tm_codes[l], 0, row, p.c * (kChunk / kSlice), &sh.full[s]);
                tma_load_3d(sh.srel[s], &a.tm_srel[l], 0, row, p.c * (kChunk / 256), &sh.full[s]);
            };
            // L2 prefetch of the weights of a stage `ahead` stages beyond the
            // shared-memory ring, so that a refill of the ring usually finds
            // its data in L2
            auto prefetch = [&](const Pos &p) {
                int l, row;
                locate<C::kRows>(a, p.tile, l, row);
                tma_prefetch_3d(&a.tm_codes[l], 0, row, p.c * (kChunk / kSlice));
                tma_prefetch_3d(&a.tm_srel[l], 0, row, p.c * (kChunk / 256));
            };
            auto acts = [&](const Pos &p, int s) {
                tma_load_3d(sh.x[s], &a.tm_x, 0, 0, p.c * (kChunk / kSlice), &sh.full[s]);
            };
            // The first stages' weights go out before the activation kernel has
            // finished; their activation copies follow the dependency wait.
            const int pre = total < STAGES ? total : STAGES;
            Pos pw{0, (int)blockIdx.x};  // the next stage to issue
            for (int q = 0; q < pre; ++q) {
                mbar_arrive_expect_tx(&sh.full[q], stage_tx);
                weights(pw, q);
                step(pw);
            }
            Pos pp = pw;  // the next stage to prefetch
            for (int q = pre; q < pre + a.ahead; ++q) {
                if (q < total)
                    prefetch(pp);
                step(pp);
            }
            asm volatile("griddepcontrol.wait;" ::: "memory");
            {
                Pos pa{0, (int)blockIdx.x};
                for (int q = 0; q < pre; ++q) {
                    acts(pa, q);
                    step(pa);
                }
            }
            int issued_upto = pre;  // stages [0, issued_upto) of the run have been issued
            bool ok = true;
            for (int q = pre; q < total; ++q) {
                const int s = q % STAGES;
                const uint32_t ph = (uint32_t)(q / STAGES) & 1u;
                if (!mbar_wait_bounded(&sh.empty[s], ph ^ 1u, abort)) {
                    ok = false;
                    issued_upto = q;
                    break;
                }
                mbar_arrive_expect_tx(&sh.full[s], stage_tx);
                weights(pw, s);
                acts(pw, s);
                step(pw);
                if (q + a.ahead < total)
                    prefetch(pp);
                step(pp);
            }
            if (!ok) {
                // let the copies in flight land before the CTA exits
                for (int q = issued_upto - STAGES < 0 ? 0 : issued_upto - STAGES; q < issued_upto; ++q) {
                    volatile int no_abort = 0;
                    mbar_wait_bounded(&sh.full[q % STAGES], (uint32_t)(q / STAGES) & 1u, &no_abort, 20000000ull);
                }
            }
        }
    } else if (warp < kConsumerWarps) {
        // ------------------------------------------------ consumers
        if (tid < 16)
            sh.cb[tid] = a.codebook[tid];
        asm volatile("bar.sync 2, %0;" ::"n"(kThreads) : "memory");
        {
            // the plain level table of scale byte tid, or its split form
            const uint4 e = lut_entry((uint32_t)tid, sh.cb);
            bool split_ok;
            const uint4 t = SPLIT ? lut_entry_split(e, split_ok) : e;
#pragma unroll
            for (int r = 0; r < C::kCopies; ++r)
                sh.lut[tid * C::kCopies + ((r + tid) & (C::kCopies - 1))] = t;
        }
        consumer_sync();
        // (the consumers read only shared memory: the activation copies
        // already wait for the previous kernel in the producer)

        const int g = lane >> 2, t = lane & 3, sl = warp;
        const uint8_t *lutb = reinterpret_cast<const uint8_t *>(sh.lut + (lane & (C::kCopies - 1)));
        // this thread's offsets inside a stage (row g; g + 8 at +512 and +128;
        // MMA row block b at +1024 b and +256 b)
        const int off_code = sl * (kRows * 64) + g * 64 + 16 * t;
        const int off_srel = (sl >> 1) * (kRows * 16) + g * 16 + 8 * (sl & 1) + 2 * t;
        // 128-byte line of (slice sl, token g); the swizzle permutes the
        // 16-byte chunks of a line by its index mod 8
        const int xl = sl * M + g;
        const int off_x0 = xl * 128 + 16 * ((2 * t) ^ (xl & 7));
        const int off_x1 = xl * 128 + 16 * ((2 * t + 1) ^ (xl & 7));
        // chunks in which this warp's slice lies inside K (K is a multiple of 256)
        const int nvalid = (K - kSlice * sl + kChunk - 1) / kChunk;
        // hand a tile's partial sums to the epilogue warp and go on
        auto hand_off = [&](int seg, int32_t (&c)[kBlocks][4], int32_t (&d)[kBlocks][4]) {
            const int rb = seg % kRedBufs;
            const bool ok = mbar_wait_bounded_warp(&sh.red_empty[rb], ((uint32_t)(seg / kRedBufs) & 1u) ^ 1u, abort);
            // C fragment: c0 (row g, token 2t), c1 (g, 2t+1), c2 (g+8, 2t), c3 (g+8, 2t+1)
#pragma unroll
            for (int b = 0; b < kBlocks; ++b) {
                const int r = kMmaRows * b + g;
                sh.red[rb][warp][r][2 * t] = c[b][0] + d[b][0];
                sh.red[rb][warp][r][2 * t + 1] = c[b][1] + d[b][1];
                sh.red[rb][warp][r + 8][2 * t] = c[b][2] + d[b][2];
                sh.red[rb][warp][r + 8][2 * t + 1] = c[b][3] + d[b][3];
            }
            __syncwarp();
            if (ok && lane == 0)
                mbar_arrive(&sh.red_full[rb]);
#pragma unroll
            for (int b = 0; b < kBlocks; ++b)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    c[b][i] = d[b][i] = 0;
        };
        // two accumulators per row block break the dependency chain between MMAs
        int32_t c[kBlocks][4], d[kBlocks][4];
#pragma unroll
        for (int b = 0; b < kBlocks; ++b)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                c[b][i] = d[b][i] = 0;
        int ch = 0, seg = 0;
        // The ring is walked STAGES stages at a time with the stage index a
        // compile-time constant, so every shared-memory address is a fixed
        // offset from this thread's base registers.
        for (int q0 = 0; q0 < total; q0 += STAGES) {
            const uint32_t ph = (uint32_t)(q0 / STAGES) & 1u;
#pragma unroll
            for (int s = 0; s < STAGES; ++s) {
                if (q0 + s < total) {
                    const bool ok = mbar_wait_bounded_warp(&sh.full[s], ph, abort);
                    if (ok && ch < nvalid) {
                        Ops o[kBlocks];
                        o[0].X0 = *reinterpret_cast<const uint4 *>(sh.x[s] + off_x0);
                        o[0].X1 = *reinterpret_cast<const uint4 *>(sh.x[s] + off_x1);
#pragma unroll
                        for (int b = 0; b < kBlocks; ++b) {
                            if (b > 0) {
                                o[b].X0 = o[0].X0;
                                o[b].X1 = o[0].X1;
                            }
                            fetch_w(o[b], sh.codes[s] + off_code + 1024 * b, sh.srel[s] + off_srel + 256 * b, lutb,
                                    a.lut_step);
                        }
#pragma unroll
                        for (int b = 0; b < kBlocks; ++b) {
                            if constexpr (SPLIT)
                                slice_mma_split(o[b], c[b], d[b]);
                            else
                                slice_mma(o[b], c[b], d[b]);
                        }
                    }
                    __syncwarp();
                    if (ok && lane == 0)
                        mbar_arrive_relaxed(&sh.empty[s]);
                    if (++ch == nchunks) {
                        hand_off(seg, c, d);
                        ch = 0;
                        ++seg;
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue warp
        // Per tile: sum the eight warps' partials and write the outputs, while
        // the consumers already decode the next tile.
        asm volatile("bar.sync 2, %0;" ::"n"(kThreads) : "memory");
        asm volatile("griddepcontrol.wait;" ::: "memory");
        for (int seg = 0; seg < my_tiles; ++seg) {
            const int tile = (int)blockIdx.x + seg * (int)gridDim.x;
            int l, row0;
            locate<C::kRows>(a, tile, l, row0);
            const GemvLayer &ly = a.layer[l];
            const int N = ly.N;
            const float *__restrict__ ws = ly.ws;
            const float *__restrict__ bias = ly.bias;
            const float *__restrict__ xs = a.xs;
            void *__restrict__ out = ly.out;
            int32_t *__restrict__ acc_out = ly.acc_out;
            const bool out_f32 = a.out_f32 != 0;
            // this lane's outputs: e = lane + 32 u -> row e / 8, token e % 8
            constexpr int kOut = kRows * kTokens / 32;  // outputs per lane
            float exs[kOut], ews[kOut], eb[kOut];
            bool live[kOut];
#pragma unroll
            for (int u = 0; u < kOut; ++u) {
                const int e = lane + 32 * u, r = e >> 3, m = e & 7, n = row0 + r;
                live[u] = m < M && n < N;
                exs[u] = live[u] ? xs[m] : 0.0f;
                ews[u] = live[u] ? ws[n] : 0.0f;
                eb[u] = (live[u] && bias != nullptr) ? bias[n] : 0.0f;
            }
            const int rb = seg % kRedBufs;
            const bool ok = mbar_wait_bounded_warp(&sh.red_full[rb], (uint32_t)(seg / kRedBufs) & 1u, abort);
            int32_t acc[kOut];
#pragma unroll
            for (int u = 0; u < kOut; ++u) {
                const int e = lane + 32 * u;
                int32_t v = 0;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w)
                    v += sh.red[rb][w][e >> 3][e & 7];
                acc[u] = v;
            }
            __syncwarp();
            if (ok && lane == 0)
                mbar_arrive(&sh.red_empty[rb]);
            // warp-uniform, as the SwiGLU path shuffles across lanes
            const bool go = __shfl_sync(0xffffffffu, (int)(ok && !*abort), 0) != 0;
            if (go && ly.swiglu) {
                // rows 2f (gate) and 2f + 1 (up) of a pair are lanes l and l + 8
                // of the same u (row0 is a multiple of 16)
                const int F = N >> 1;
#pragma unroll
                for (int u = 0; u < kOut; ++u) {
                    const int e = lane + 32 * u, n = row0 + (e >> 3), m = e & 7;
                    float y = __fmul_rn(__int2float_rn(acc[u]), __fmul_rn(exs[u], ews[u]));
                    if (bias != nullptr)
                        y = __fadd_rn(y, eb[u]);
                    const float up = __shfl_down_sync(0xffffffffu, y, 8);
                    if (live[u] && ((lane >> 3) & 1) == 0) {
                        const float v = swiglu_value(y, up);
                        const int64_t o = (int64_t)m * F + (n >> 1);
                        if (out_f32)
                            reinterpret_cast<float *>(out)[o] = v;
                        else
                            reinterpret_cast<uint16_t *>(out)[o] = to_bf16_bits(v);
                    }
                }
            } else if (go && !out_f32 && acc_out == nullptr && (N & 7) == 0 && row0 + kRows <= N) {
                // a whole tile of bf16 outputs: staged token-major, then each
                // token's kRows outputs leave as kRows / 8 16-byte stores
#pragma unroll
                for (int u = 0; u < kOut; ++u) {
                    const int e = lane + 32 * u;
                    float y = __fmul_rn(__int2float_rn(acc[u]), __fmul_rn(exs[u], ews[u]));
                    if (bias != nullptr)
                        y = __fadd_rn(y, eb[u]);
                    sh.ostage[e & 7][e >> 3] = to_bf16_bits(y);
                }
                __syncwarp();
                constexpr int kPieces = kRows / 8;  // 16-byte pieces of a token's outputs
                if (lane < kPieces * M) {
                    const int m = lane / kPieces, h = lane % kPieces;
                    const uint4 v = *reinterpret_cast<const uint4 *>(&sh.ostage[m][8 * h]);
                    *reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(out) + (int64_t)m * N + row0 + 8 * h) = v;
                }
                __syncwarp();
            } else if (go) {
#pragma unroll
                for (int u = 0; u < kOut; ++u) {
                    if (!live[u])
                        continue;
                    const int e = lane + 32 * u, n = row0 + (e >> 3), m = e & 7;
                    float y = __fmul_rn(__int2float_rn(acc[u]), __fmul_rn(exs[u], ews[u]));
                    if (bias != nullptr)
                        y = __fadd_rn(y, eb[u]);
                    const int64_t o = (int64_t)m * N + n;
                    if (out_f32)
                        reinterpret_cast<float *>(out)[o] = y;
                    else
                        reinterpret_cast<uint16_t *>(out)[o] = to_bf16_bits(y);
                    if (acc_out != nullptr)
                        acc_out[o] = acc[u];
                }
            }
        }
    }
    __syncthreads();
}

// Whether every scale byte of a layer has a split table (lut_entry_split)
// for this codebook: each CTA tabulates the 256 bytes' split forms, takes
// tmin = the smallest magnitude (s & 0x7F) without one, and flags (in *bad,
// which the host zeroed) any byte of its rows of srel [N, K / 16] with
// s & 0x7F >= tmin.  Bytes below tmin all have a split form by its
// definition; above it some may too (the check is conservative).  Per 4
// bytes, bit 7 of each byte of (w & 0x7F7F7F7F) + (128 - tmin) * 0x01010101 is
// set iff that byte's magnitude is >= tmin (no carry crosses a byte).
__global__ void __launch_bounds__(256) split_check_kernel(const uint8_t *__restrict__ srel, int64_t bytes,
                                                          const float *__restrict__ codebook, int *__restrict__ bad)
{
    __shared__ float cb[16];
    __shared__ int tmin;
    if (threadIdx.x < 16)
        cb[threadIdx.x] = codebook[threadIdx.x];
    if (threadIdx.x == 0)
        tmin = 128;
    __syncthreads();
    bool ok;
    lut_entry_split(lut_entry(threadIdx.x, cb), ok);
    if (!ok)
        atomicMin(&tmin, (int)(threadIdx.x & 0x7Fu));
    __syncthreads();
    const uint32_t addc = (uint32_t)(128 - tmin) * 0x01010101u;
    uint32_t flags = 0u;
    const int64_t words = bytes / 16;  // whole 16-byte pieces (K / 16 is a multiple of 16)
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < words; i += (int64_t)gridDim.x * blockDim.x) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(srel) + i);
        flags |= (((v.x & 0x7F7F7F7Fu) + addc) | ((v.y & 0x7F7F7F7Fu) + addc) | ((v.z & 0x7F7F7F7Fu) + addc) |
                  ((v.w & 0x7F7F7F7Fu) + addc)) & 0x80808080u;
    }
    if (__syncthreads_or(flags != 0u) && threadIdx.x == 0)
        atomicOr(bad, 1);
}

}  // namespace gv
}  // namespace cr
