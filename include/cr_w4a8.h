/*
 * cr_w4a8.h -- C ABI of the ConvRot W4A8 codebook linear layer forward on
 * NVIDIA B200 (sm_100a).
 *
 * The layer (ai-toolkit convrot_w4a8_quant.py, module docstring) stores a
 * linear weight W [N out, K in] that was rotated by a block regular Hadamard
 * (block R = 256) as 4-bit codebook indices with one fp8 e4m3fn relative
 * scale per group of G = 16 columns and one fp32 scale per output channel:
 *
 *   w_int8[n, k] = sat_s8(rne(codebook[code[n, k]] * s_rel[n, k / 16]))
 *   W_rot[n, k]  = w_int8[n, k] * s_channel[n]
 *
 * The forward rotates each activation row block-wise by the same Hadamard,
 * quantises it per token to int8, contracts int8 x int8 -> int32 and rescales
 * by the per-token and per-channel scales:
 *
 *   y[m, n] = bf16( float(sum_k xq[m, k] * w_int8[n, k]) * (xs[m] * s_channel[n]) [+ bias[n]] )
 *
 * Conventions for every entry point
 * ---------------------------------
 * - Pointers are DEVICE pointers unless stated otherwise; the caller owns
 *   every buffer it passes.  Every call is asynchronous on `stream` (NULL =
 *   the legacy default stream) and returns as soon as the work is queued.
 * - Device memory of the library.  The prefill paths need a weight
 *   transient: cr_w4a8_gemm, cr_w4a8_gemm_swiglu, and cr_w4a8_linear,
 *   cr_w4a8_linear_swiglu, cr_w4a8_linear_grouped and cr_w4a8_plan_forward
 *   when M > 8, take N * K bytes (the int8 weight; grouped: the largest
 *   layer's) and cr_w4a8_ste_backward 2 * N * K bytes (the transposed bf16
 *   weight) from a stream-ordered pool of the library, allocated on `stream`
 *   and freed on it at the end of the call.  The pool keeps nothing: its
 *   memory goes back to the driver at the next stream, event or device
 *   synchronisation after the free.  When that allocation fails the call
 *   returns CR_ERR_CUDA and launches nothing.  The *_ws variants
 *   (cr_w4a8_gemm_ws, cr_w4a8_linear_ws, cr_w4a8_ste_backward_ws) take the
 *   transient from the caller instead and allocate nothing; every other entry
 *   point allocates no device memory.
 * - cr_w4a8_linear (and _swiglu, _ws, _grouped, cr_w4a8_plan_forward) with
 *   M > 8 run the weight decode on a side stream of the library (one
 *   non-blocking stream and two events per device, created on first use and
 *   kept until exit), forked from and joined back into `stream` with events,
 *   so the decode overlaps the activation kernel; `stream` orders the call
 *   as usual.
 * - Arrays are dense and row-major, with exactly the shapes given.
 * - Every pointer must be 16-byte aligned (CR_ERR_ALIGNMENT otherwise).
 * - Sizes are int64_t.  M == 0 or N == 0 is an empty problem: CR_OK, nothing
 *   is launched.  Negative sizes give CR_ERR_INVALID_ARG.
 * - K must be a positive multiple of 256 (the rotation block; it implies the
 *   group size 16) and at most CR_MAX_K (CR_ERR_UNSUPPORTED otherwise).
 * - Arguments are validated before anything is launched; a failed validation
 *   launches nothing and leaves every output untouched.  Launch failures
 *   return CR_ERR_CUDA.  Nothing falls back to another implementation.
 * - Values are not validated: activations must be finite with |x| < 2^119,
 *   so that no partial sum of the block rotation (at most 256 |x|) overflows
 *   fp32; for other values the outputs are unspecified, but no call faults.
 * - Calls that read a buffer another call on another stream is writing race,
 *   as with any CUDA kernel.
 * - Overlapped launches.  cr_rotate_quant_act, cr_w4a8_gemv, cr_w4a8_linear
 *   (decode path) and cr_w4a8_linear_decode_noalloc launch their kernels as
 *   programmatic dependents of the previous kernel on the stream, and those
 *   kernels allow the next kernel to launch early.  Stream order still holds
 *   for every activation, scale and output buffer: each kernel waits for its
 *   predecessor to complete before it reads a result of it or writes a
 *   buffer that the predecessor may read.  The decode GEMV alone starts
 *   reading the layer (qdata, srel, codebook) before that wait, so the layer
 *   must not be written by a kernel that itself allows early launch of its
 *   dependents (griddepcontrol.launch_dependents / PDL) and immediately
 *   precedes the GEMV on the stream; a kernel that does not, and every copy
 *   or memset, orders as usual.
 */
#ifndef CR_W4A8_H
#define CR_W4A8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (the same handle type, declared without the CUDA headers). */
typedef struct CUstream_st *cr_stream_t;

typedef enum {
    CR_OK = 0,
    CR_ERR_INVALID_ARG = 1,  /* null pointer, negative size, MP < M, act_qmax outside 1..127 */
    CR_ERR_UNSUPPORTED = 2,  /* K not a positive multiple of 256, K > CR_MAX_K, GEMV with M > 8 */
    CR_ERR_ALIGNMENT = 3,    /* a pointer is not 16-byte aligned */
    CR_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    CR_ERR_TIMEOUT = 5,      /* a kernel gave up waiting on its own pipeline (see cr_check_device_error) */
    CR_ERR_NO_DEVICE = 6     /* no sm_100 device is current */
} cr_status;

typedef enum {
    CR_OUT_BF16 = 0, /* output elements are bf16, rounded to nearest even */
    CR_OUT_F32 = 1   /* output elements are fp32 */
} cr_out_dtype;

/* Largest supported K: keeps |acc| <= 127 * 128 * K inside int32
 * (ai-toolkit convrot_w4a8_quant.py, w4a8_gemv_kernel: int32 accumulation). */
#define CR_MAX_K 131072
/* Rotation block and group size (ai-toolkit convrot_w4a8_quant.py,
 * ConvRotW4A8Quantizer.__init__ defaults rot_size=256, group_size=16). */
#define CR_ROT 256
#define CR_GROUP 16
/* Largest M the decode GEMV takes (ai-toolkit convrot_w4a8_quant.py,
 * W4A8_GEMV_MAX_M). */
#define CR_GEMV_MAX_M 8

/* Static, NUL-terminated description of a status code.  Host only. */
const char *cr_status_string(cr_status s);

/*
 * (1) Rotate + per-token int8 quantisation of the activations.
 *
 * Defined by: ai-toolkit convrot_w4a8_quant.py, prepare_act (rotate, then
 * quantise the rows once) and w4a8_act_quant_kernel (per-row symmetric int8
 * quant into exactly MP rows); the rotation is h3-rs src/weights.rs,
 * hadamard() / rotate_activation(): each 256-column block of a row times
 * H_256 = (h4 (x) h4 (x) h4 (x) h4) / 16.
 *
 *   r      = x rotated block-wise, in fp32 from the exact bf16 inputs, digit
 *            stages in the order stride 1, 4, 16, 64; per quadruple
 *            out[a] = ((v0 + v1) + (v2 + v3)) - 2 * v[3 - a]; then * 1/16
 *   xs[m]  = max_k |r[m, k]| / act_qmax   (1.0 if that max is 0)
 *   xq[m,k]= clamp(rint(r[m, k] / xs[m]), -act_qmax, act_qmax)
 *   rows M <= m < MP:  xq = 0, xs = 1
 *
 * x   [M, K]  bf16 (bit patterns), read only.
 * xq  [MP, K] int8, written.     xs [MP] fp32, written.
 * MP >= M (the decode GEMV pads to the next power of two; prefill passes MP = M).
 * act_qmax in 1..127 (the layer uses 127).
 */
cr_status cr_rotate_quant_act(const uint16_t *x, int64_t M, int64_t K, int64_t MP,
                              int act_qmax, int8_t *xq, float *xs, cr_stream_t stream);

/*
 * (2) Decode the packed codes onto the int8 grid.
 *
 * Defined by: ai-toolkit convrot_w4a8_quant.py, module docstring storage
 * formula, unpack_w4a8_eager and w4a8_unpack_kernel with W4A8_SAT = True:
 *   w8[n, k] = sat_s8(rne(codebook[code(n, k)] * fp8(srel[n, k / 16])))
 * where code(n, 2j) is the low nibble and code(n, 2j+1) the high nibble of
 * qdata[n, j], the product is one fp32 multiply, rne rounds to nearest even
 * and sat_s8 saturates to [-128, 127] (a NaN product gives 0).
 *
 * qdata    [N, K/2]  packed codes, read only.
 * srel     [N, K/16] fp8 e4m3fn scale bytes, read only.
 * codebook [16]      fp32 levels, read only.
 * w8       [N, K]    int8, written.
 */
cr_status cr_w4a8_decode_int8(const uint8_t *qdata, const uint8_t *srel, const float *codebook,
                              int64_t N, int64_t K, int8_t *w8, cr_stream_t stream);

/*
 * (3) Prefill forward for any M: decode + int8 tensor-core contraction +
 * epilogue.
 *
 * Defined by: ai-toolkit convrot_w4a8_quant.py, _w4a8_linear_ste_op (decode
 * the codes, quantise the activations, torch._int_mm(aq, w8.t()), then
 * _int8_epilogue) with the epilogue of w4a8_gemv_kernel:
 *   acc[m, n] = sum_k xq[m, k] * w8[n, k]          (exact int32)
 *   out[m, n] = float(acc) * (xs[m] * s_channel[n]) [+ bias[n]], each op
 *               rounded on its own, then cast to out_dtype.
 *
 * xq        [M, K] int8 and xs [M] fp32: the output of cr_rotate_quant_act.
 * qdata, srel, codebook: as in cr_w4a8_decode_int8.
 * s_channel [N] fp32.   bias [N] fp32, or NULL for no bias.
 * out       [M, N] bf16 or fp32 per out_dtype, written.
 * acc_out   [M, N] int32, or NULL: when given, the raw accumulators are
 *           written too (a parity/debug output).
 */
cr_status cr_w4a8_gemm(const int8_t *xq, const float *xs, const uint8_t *qdata, const uint8_t *srel,
                       const float *codebook, const float *s_channel, const float *bias,
                       int64_t M, int64_t N, int64_t K, cr_out_dtype out_dtype, void *out,
                       int32_t *acc_out, cr_stream_t stream);

/*
 * (3w) (3) with the caller's weight transient: w8_work [N, K] int8 (16-byte
 * aligned, required unless M == 0 or N == 0) receives the decoded weight (the
 * int8 grid of (2)) and is then read by the contraction; on return it holds
 * that grid.  Allocates nothing.  Results equal those of (3) bit for bit.
 */
cr_status cr_w4a8_gemm_ws(const int8_t *xq, const float *xs, const uint8_t *qdata, const uint8_t *srel,
                          const float *codebook, const float *s_channel, const float *bias,
                          int64_t M, int64_t N, int64_t K, cr_out_dtype out_dtype, void *out,
                          int32_t *acc_out, int8_t *w8_work, cr_stream_t stream);

/*
 * (4) Decode forward for 1 <= M <= 8: a fused GEMV that streams the packed
 * codes, the fp8 group scales and the codebook (4.5 bits per weight) and
 * never materialises the int8 weight.
 *
 * Defined by: ai-toolkit convrot_w4a8_quant.py, w4a8_gemv_kernel and
 * gemv_prepared.  Same arguments and the same results as cr_w4a8_gemm,
 * bit for bit (int32 accumulation is exact and order independent, and both
 * share the epilogue).  xq needs only its first M rows.  M > 8 gives
 * CR_ERR_UNSUPPORTED.
 */
cr_status cr_w4a8_gemv(const int8_t *xq, const float *xs, const uint8_t *qdata, const uint8_t *srel,
                       const float *codebook, const float *s_channel, const float *bias,
                       int64_t M, int64_t N, int64_t K, cr_out_dtype out_dtype, void *out,
                       int32_t *acc_out, cr_stream_t stream);

/*
 * (5) The epilogue alone, on an int32 accumulator.
 *
 * Defined by: ai-toolkit convrot_w4a8_quant.py, w4a8_gemv_kernel epilogue
 * (and _int8_epilogue, called with the same arguments by the prefill op):
 *   out[m, n] = float(acc[m, n]) * (xs[m] * s_channel[n]) [+ bias[n]]
 *
 * acc [M, N] int32, xs [M] fp32, s_channel [N] fp32, bias [N] fp32 or NULL;
 * out [M, N] bf16 or fp32, written.
 */
cr_status cr_epilogue(const int32_t *acc, const float *xs, const float *s_channel, const float *bias,
                      int64_t M, int64_t N, cr_out_dtype out_dtype, void *out, cr_stream_t stream);

/*
 * (6) The whole layer forward in one call: (1), then (4) when M <= 8, else (3).
 *
 * Defined by: ai-toolkit convrot_w4a8_quant.py, ConvRotW4A8Quantizer.forward
 * (decode GEMV when gemv_ok, otherwise the prefill op).
 *
 * x [M, K] bf16 bits; weights as in (3); out [M, N].
 * xq_work [max(M, MP), K] int8 and xs_work [max(M, MP)] fp32 are caller-owned
 * scratch for the quantised activations, where MP is the next power of two
 * of M when M <= 8 and M otherwise; their contents on return are the
 * quantised activations.
 */
cr_status cr_w4a8_linear(const uint16_t *x, const uint8_t *qdata, const uint8_t *srel,
                         const float *codebook, const float *s_channel, const float *bias,
                         int64_t M, int64_t N, int64_t K, int act_qmax, cr_out_dtype out_dtype,
                         void *out, int8_t *xq_work, float *xs_work, cr_stream_t stream);

/*
 * (6w) (6) with the caller's weight transient for the prefill path: when
 * M > 8, w8_work [N, K] int8 (16-byte aligned; CR_ERR_INVALID_ARG if NULL)
 * receives the decoded weight, as in (3w); when M <= 8 it is not used and may
 * be NULL.  Allocates nothing.  Results equal those of (6) bit for bit.
 */
cr_status cr_w4a8_linear_ws(const uint16_t *x, const uint8_t *qdata, const uint8_t *srel,
                            const float *codebook, const float *s_channel, const float *bias,
                            int64_t M, int64_t N, int64_t K, int act_qmax, cr_out_dtype out_dtype,
                            void *out, int8_t *xq_work, float *xs_work, int8_t *w8_work, cr_stream_t stream);

/*
 * (7) The decode forward (1 <= M <= 8) without any allocation.
 *
 * The pages have no counterpart of this entry point; it exists for callers
 * that cannot allocate device memory at the time of the call and so cannot
 * supply the scratch buffers cr_w4a8_linear needs: serving loops whose device
 * memory is all owned by their own allocator (nothing is left to carve
 * scratch from), and real-time paths that cannot afford the synchronisation
 * an allocation can imply.
 *
 * It computes exactly what cr_w4a8_linear computes for M <= 8 (rotate +
 * quantise, then the decode GEMV), with the quantised activations kept in a
 * scratch array that the library reserves statically on every device that
 * loads it (CR_NOALLOC_SCRATCH_BYTES, held until the process exits).  The
 * caller still passes x, the layer and out, as for cr_w4a8_linear.
 *
 * Limits: 1 <= M <= 8 and K <= CR_MAX_K, so the padded activations
 * (next power of two of M rows x K bytes) always fit; M > 8 returns
 * CR_ERR_UNSUPPORTED.  It calls no allocation routine.
 * The first call on a device looks up the scratch array's device address;
 * make that first call before any stream capture on that device.
 * Every call on a device shares the one scratch array, so calls whose
 * kernels overlap on the GPU (different streams, or concurrent host threads)
 * race and give undefined results; serialise them on one stream.
 */
#define CR_NOALLOC_SCRATCH_BYTES (CR_GEMV_MAX_M * CR_MAX_K + 256)
cr_status cr_w4a8_linear_decode_noalloc(const uint16_t *x, const uint8_t *qdata, const uint8_t *srel,
                                        const float *codebook, const float *s_channel, const float *bias,
                                        int64_t M, int64_t N, int64_t K, int act_qmax, cr_out_dtype out_dtype,
                                        void *out, cr_stream_t stream);

/*
 * (8) Several layers fed the same input, in one decode launch.
 *
 * Defined by: ai-toolkit convrot_w4a8_quant.py, w4a8_grouped_linear (layers
 * that share the rotation share one rotate + quantise of x on the decode
 * path) and gemv_prepared for each layer.  Here the layers' GEMVs are also one
 * launch: their row tiles are numbered one after the other and spread over
 * one persistent grid, so small layers (q/k/v, gate/up) share one ramp-up and
 * one tail.  Every layer's outputs equal those of cr_w4a8_gemv on that layer,
 * bit for bit.
 *
 * cr_w4a8_layer (all pointers device pointers, 16-byte aligned):
 *   qdata [N, K/2], srel [N, K/16], s_channel [N], bias [N] or NULL,
 *   out [M, N] (bf16 or fp32 as out_dtype), acc_out [M, N] int32 or NULL.
 *   N >= 0 (N == 0: the layer produces nothing).
 * All layers use the same K, the same codebook[16] (the one they were
 * quantised with; the pages' fixed codebook) and the same activations.
 * 1 <= num_layers <= CR_MAX_LAYERS, else CR_ERR_INVALID_ARG; `layers` is a
 * host array, read during the call only.
 */
#define CR_MAX_LAYERS 4
typedef struct {
    const uint8_t *qdata;
    const uint8_t *srel;
    const float *s_channel;
    const float *bias;
    int64_t N;
    void *out;
    int32_t *acc_out;
} cr_w4a8_layer;

/* (8a) The grouped decode GEMV on quantised activations (xq [>= M, K] int8,
 * xs [M] fp32), 1 <= M <= 8; M > 8 gives CR_ERR_UNSUPPORTED. */
cr_status cr_w4a8_gemv_grouped(const int8_t *xq, const float *xs, const float *codebook, int64_t M, int64_t K,
                               const cr_w4a8_layer *layers, int num_layers, cr_out_dtype out_dtype,
                               cr_stream_t stream);

/* (8b) The grouped layer forward: (1) once, then (8a) when M <= 8, or (3)
 * for each layer when M > 8.  x, xq_work, xs_work as in (6); acc_out must be
 * NULL in every layer (CR_ERR_INVALID_ARG otherwise). */
cr_status cr_w4a8_linear_grouped(const uint16_t *x, const float *codebook, int64_t M, int64_t K,
                                 const cr_w4a8_layer *layers, int num_layers, int act_qmax,
                                 cr_out_dtype out_dtype, int8_t *xq_work, float *xs_work, cr_stream_t stream);

/*
 * (9) SwiGLU fused into the epilogue, for a gate/up layer whose output rows
 * are interleaved.
 *
 * Defined by: h3-rs src/weights.rs, QLinear::interleave_swiglu (the gate and
 * up projections' output rows reordered to pairs g0, u0, g1, u1, ... so the
 * activation fuses into the int8 GEMM), swiglu_interleaved and run_swiglu
 * (silu(gate) * up over each pair).
 *
 * The layer holds N = 2F rows in that order (cr_interleave_rows builds it
 * from the two halves [gate; up]).  With g and u the fp32 epilogue values of
 * rows 2f and 2f + 1, computed exactly as in (3),
 *   out[m, f] = out_dtype( silu(g) * u ),  silu(g) = g / (1 + exp(-g))
 * in fp32: with t = expf(-|g|), silu(g) = g / (1 + t) for g >= 0 and
 * g * t / (1 + t) for g < 0 (the same value, and no overflow for very
 * negative gates), the division by the fast __fdividef (at most 2 ulp for a
 * divisor in [1, 2]), each op rounded on its own, then rounded once to
 * out_dtype.  out is [M, F]; N odd gives CR_ERR_INVALID_ARG.  There
 * is no acc_out: the int32 accumulators are those of (3) and (4) on the same
 * layer.  The decode GEMV and the GEMM give the same bits.
 *
 * (9a) on quantised activations, any M (the prefill GEMM of (3));
 * (9b) on quantised activations, 1 <= M <= 8 (the decode GEMV of (4));
 * (9c) the whole forward as (6).
 */
cr_status cr_w4a8_gemm_swiglu(const int8_t *xq, const float *xs, const uint8_t *qdata, const uint8_t *srel,
                              const float *codebook, const float *s_channel, const float *bias,
                              int64_t M, int64_t N, int64_t K, cr_out_dtype out_dtype, void *out,
                              cr_stream_t stream);
cr_status cr_w4a8_gemv_swiglu(const int8_t *xq, const float *xs, const uint8_t *qdata, const uint8_t *srel,
                              const float *codebook, const float *s_channel, const float *bias,
                              int64_t M, int64_t N, int64_t K, cr_out_dtype out_dtype, void *out,
                              cr_stream_t stream);
cr_status cr_w4a8_linear_swiglu(const uint16_t *x, const uint8_t *qdata, const uint8_t *srel,
                                const float *codebook, const float *s_channel, const float *bias,
                                int64_t M, int64_t N, int64_t K, int act_qmax, cr_out_dtype out_dtype,
                                void *out, int8_t *xq_work, float *xs_work, cr_stream_t stream);

/*
 * (10) Row interleave of a gate/up layer's arrays.
 *
 * Defined by: h3-rs src/weights.rs, interleave_rows: rows [0, F) and
 * [F, 2F) of src become pairs, dst row 2f = src row f and dst row 2f + 1 =
 * src row F + f, each row `row_bytes` bytes.  Apply it to qdata (K/2 bytes a
 * row), srel (K/16), s_channel (4) and bias (4) of the stacked [gate; up]
 * layer to get the layout (9) reads.  A one-time preparation, not part of the
 * forward.
 *
 * src, dst: device buffers of rows * row_bytes bytes that must not overlap
 * (CR_ERR_INVALID_ARG otherwise); no alignment is required.  rows must be even
 * (CR_ERR_INVALID_ARG otherwise); rows == 0 or row_bytes == 0 does nothing.
 */
cr_status cr_interleave_rows(const void *src, void *dst, int64_t rows, int64_t row_bytes, cr_stream_t stream);

/*
 * (11) Offline quantiser: rotated fp32 weights -> the layer's storage.
 *
 * Defined by: ai-toolkit convrot_w4a8_quant.py, quantize_w4a8_rotated and
 * _quantize_rotated_rows, with _assign_codes, grid_levels and _assign_grid
 * (deterministic) and _ALS_ITERS = 2.  Per row n and group g of 16 columns,
 * with "nearest" the pages' rule (search the sorted table, compare the fp32
 * distances to the two neighbours, the upper one only when strictly nearer):
 *   gs     = clamp(max |w|, 1e-8); codes = nearest codebook index of w / gs
 *   twice: lv = codebook[codes];
 *          gs = clamp(sum(w * lv) / clamp(sum(lv * lv), 1e-8), 1e-8);
 *          codes = nearest codebook index of w / gs
 *   s_channel[n] = clamp(max over the row of |codebook[code] * gs| / 127, 1e-8)
 *   srel[n, g]   = fp8_e4m3fn(gs / s_channel[n])  (nearest, ties to even;
 *                  a magnitude rounding above 448 gives NaN, as torch's cast)
 *   final code   = nearest level of w / s_channel[n] among
 *                  clamp(rint(codebook[i] * fp8(srel[n, g])), -127, 127)
 * Every operation is one IEEE fp32 operation; each sum of 16 products is
 * taken pairwise, ((p0 + p1) + (p2 + p3)) + ... (the pages leave that order
 * open).
 *
 * w_rot [N, K] fp32 (the weight already rotated block-wise), codebook [16]
 * sorted ascending; qdata [N, K/2], srel [N, K/16] (fp8 bytes) and
 * s_channel [N] are written.  K must be a positive multiple of 16, at most
 * CR_MAX_K (CR_ERR_UNSUPPORTED otherwise); N == 0 does nothing.  The weights
 * must be finite.
 */
cr_status cr_w4a8_quantize_rotated(const float *w_rot, const float *codebook, int64_t N, int64_t K,
                                   uint8_t *qdata, uint8_t *srel, float *s_channel, cr_stream_t stream);

/*
 * (12) New codes on stored scales.
 *
 * Defined by: ai-toolkit convrot_w4a8_quant.py, requantize_codes_ (after its
 * rotation) and _assign_grid.  target = w_rot[n, k] / s_channel[n] on the
 * levels clamp(rint(codebook[i] * fp8(srel[n, k / 16])), -127, 127):
 *   rand == NULL: the nearest level, as in (11);
 *   otherwise the stochastic choice: with lo the lower level of the bracket
 *     around target (lo = clamp(pos - 1, 0, 14)), the upper level when
 *     target > rand[n, k] * (level[lo + 1] - level[lo]) + level[lo]
 *     (a multiply, then an add), so that the expected level is the target.
 * rand [N, K] fp32 uniform draws in [0, 1) are an input (the caller owns the
 * random numbers).  qdata [N, K/2] is written; shapes and K as in (11).
 */
cr_status cr_w4a8_assign_codes(const float *w_rot, const uint8_t *srel, const float *s_channel,
                               const float *codebook, const float *rand, int64_t N, int64_t K,
                               uint8_t *qdata, cr_stream_t stream);

/*
 * (13) Straight-through backward: the gradient of the layer's input.
 *
 * Defined by: ai-toolkit convrot_w4a8_quant.py, _w4a8_linear_ste_backward
 * (the training path keeps only the packed codes and decodes them again in
 * the backward):
 *   w[n, k]  = bf16( w8[n, k] * bf16(s_channel[n]) )   (w8 as in (2); the
 *              product is exact in fp32 and rounded once to bf16)
 *   dx[m, k] = bf16( sum_n grad[m, n] * w[n, k] )       (fp32 accumulation)
 * dx is the gradient with respect to the layer's (rotated) input, as the
 * pages' operator returns it; the rotation's own backward is the caller's.
 *
 * grad [M, N] bf16 bits, dx [M, K] bf16 bits (written); the layer as in (3).
 * K as for the forward; N must be a multiple of 8 (CR_ERR_UNSUPPORTED
 * otherwise).  N == 0 writes dx = 0.  Internally the transposed weight (13a)
 * is built in a transient of 2 N K bytes and contracted on the tensor cores
 * (bf16 x bf16 -> fp32).
 *
 * (13a) The transposed backward weight alone: wt [K, N] bf16 bits,
 * wt[k, n] = w[n, k].
 */
cr_status cr_w4a8_ste_backward(const uint16_t *grad, const uint8_t *qdata, const uint8_t *srel,
                               const float *codebook, const float *s_channel, int64_t M, int64_t N, int64_t K,
                               uint16_t *dx, cr_stream_t stream);
cr_status cr_w4a8_dequant_t_bf16(const uint8_t *qdata, const uint8_t *srel, const float *codebook,
                                 const float *s_channel, int64_t N, int64_t K, uint16_t *wt, cr_stream_t stream);
/* (13w) (13) with the caller's transient: wt_work [K, N] bf16 (16-byte
 * aligned; CR_ERR_INVALID_ARG if NULL when M > 0 and N > 0) receives the
 * transposed weight of (13a).  Allocates nothing; dx equals that of (13). */
cr_status cr_w4a8_ste_backward_ws(const uint16_t *grad, const uint8_t *qdata, const uint8_t *srel,
                                  const float *codebook, const float *s_channel, int64_t M, int64_t N, int64_t K,
                                  uint16_t *dx, uint16_t *wt_work, cr_stream_t stream);

/*
 * (14) A prepared layer for repeated forwards (serving loops).
 *
 * The same computation as (6) for one layer, with its arguments checked and
 * the decode GEMV's weight tensor maps encoded once, at plan creation; the
 * activation map is re-encoded only when the work buffer or M changes.  The
 * pages' ConvRotW4A8Quantizer likewise prepares a layer's buffers once
 * (attach_) and reuses them on every forward.
 *
 * cr_w4a8_plan_create: the layer as in (3), act_qmax and out_dtype as in (6);
 *   the buffers must stay valid and unchanged while the plan exists.  The plan
 *   belongs to the device current at creation; *plan is written.  Creation
 *   reads the layer's scale bytes and the codebook once on the device (a check
 *   kernel on the legacy default stream, waited for before the call returns):
 *   when every scale byte's level table has the split form of the decode GEMV
 *   (two tables whose byte-permute results add up to the level; it exists
 *   unless a level of 127 pairs with a negative one), the plan's decode
 *   forwards may use that faster decode.  Results are the same bit for bit.
 * cr_w4a8_plan_forward: (6) on that device with the plan's layer: x [M, K]
 *   bf16, out [M, N], xq_work / xs_work as in (6).  Calls on one plan may come
 *   from several host threads.
 * cr_w4a8_plan_forward_host: the same with x and out in HOST memory (pinned
 *   memory lets the copies run asynchronously): queues the copy of x_host
 *   [M, K] into x_dev, the forward into out_dev [M, N], and the copy of out_dev
 *   into out_host, all on `stream`; out_host is valid once the stream has
 *   reached that point, and x_host must stay unchanged until then.  x_dev,
 *   out_dev, xq_work and xs_work are device buffers of the caller.  A copy of
 *   at most 1 MiB whose host buffer is page-locked memory mapped for the
 *   device (cudaHostAlloc, cudaMallocHost, or cudaHostRegister with mapping;
 *   every such allocation under unified addressing), 16-byte aligned and a
 *   multiple of 16 bytes long, is done by a kernel of the library on the SMs
 *   (a decode step's few tens of KB cost far less that way than a copy-engine
 *   transfer between two kernels); other copies use cudaMemcpyAsync.  The
 *   kernel copying x_host reads it before the previous kernel on the stream
 *   has finished: x_host must not be written by a kernel that immediately
 *   precedes this call and allows early launch of its dependents.  For a
 *   decode batch (M <= CR_GEMV_MAX_M) with bf16 outputs, N a multiple of 8,
 *   and an out_host that qualifies for the kernel copy, the decode GEMV
 *   stores y into out_host itself and out_dev is not written; otherwise
 *   out_dev holds y after the call.
 * cr_w4a8_plan_gemv: the decode GEMV of (4) on the plan's layer and already
 *   quantised activations (ai-toolkit convrot_w4a8_quant.py, gemv_prepared):
 *   xq [>= M, K] int8, xs [M] fp32, 1 <= M <= 8 (CR_ERR_UNSUPPORTED above),
 *   out [M, N]; the same results as cr_w4a8_gemv.
 * cr_w4a8_plan_destroy: frees the plan (NULL is allowed).
 * Errors as in (6); a plan used on another device gives CR_ERR_INVALID_ARG.
 */
typedef struct cr_w4a8_plan_st *cr_w4a8_plan;
cr_status cr_w4a8_plan_create(const uint8_t *qdata, const uint8_t *srel, const float *codebook,
                              const float *s_channel, const float *bias, int64_t N, int64_t K, int act_qmax,
                              cr_out_dtype out_dtype, cr_w4a8_plan *plan);
cr_status cr_w4a8_plan_forward(cr_w4a8_plan plan, const uint16_t *x, int64_t M, void *out, int8_t *xq_work,
                               float *xs_work, cr_stream_t stream);
cr_status cr_w4a8_plan_forward_host(cr_w4a8_plan plan, const uint16_t *x_host, int64_t M, void *out_host,
                                    uint16_t *x_dev, void *out_dev, int8_t *xq_work, float *xs_work,
                                    cr_stream_t stream);
cr_status cr_w4a8_plan_gemv(cr_w4a8_plan plan, const int8_t *xq, const float *xs, int64_t M, void *out,
                            cr_stream_t stream);
cr_status cr_w4a8_plan_destroy(cr_w4a8_plan plan);

/*
 * (17) A host-buffer forward bound to its buffers (serving loops that call
 * the same layer with the same buffers again and again).
 *
 * cr_w4a8_plan_bind_host: checks the arguments of cr_w4a8_plan_forward_host
 *   once (with the same meaning), decides each copy's path (kernel or copy
 *   engine, as there) and prepares the decode GEMV's complete arguments;
 *   *call is written (NULL on error).  The plan and every buffer must stay
 *   valid, and the host buffers page-locked, while the call exists.
 * cr_w4a8_host_call_run: queues exactly what cr_w4a8_plan_forward_host with
 *   those arguments queues (results bit for bit the same), without checking
 *   or resolving anything again; only the current device is checked
 *   (CR_ERR_INVALID_ARG if it is not the plan's).
 * cr_w4a8_host_call_destroy: frees the call (NULL is allowed); the plan and
 *   the buffers are not touched.
 */
typedef struct cr_w4a8_host_call_st *cr_w4a8_host_call;
cr_status cr_w4a8_plan_bind_host(cr_w4a8_plan plan, const uint16_t *x_host, int64_t M, void *out_host,
                                 uint16_t *x_dev, void *out_dev, int8_t *xq_work, float *xs_work,
                                 cr_w4a8_host_call *call);
cr_status cr_w4a8_host_call_run(cr_w4a8_host_call call, cr_stream_t stream);
cr_status cr_w4a8_host_call_destroy(cr_w4a8_host_call call);

/*
 * (16) The prefill contraction on an int8 weight already on the grid.
 *
 * Defined by: ai-toolkit convrot_w4a8_quant.py, _w4a8_linear_ste_op after
 * its unpack: torch._int_mm(aq, w8.t()) and the epilogue, i.e. (3) without
 * the decode.  w8 [N, K] int8 (from (2), or a weight a caller keeps decoded
 * across calls, trading 8 bits per weight of memory for the decode); the
 * other arguments as in (3), and the results equal those of (3) on the same
 * layer bit for bit.
 */
cr_status cr_gemm_s8(const int8_t *xq, const float *xs, const int8_t *w8, const float *s_channel,
                     const float *bias, int64_t M, int64_t N, int64_t K, cr_out_dtype out_dtype, void *out,
                     int32_t *acc_out, cr_stream_t stream);

/*
 * (15) Self-test of the failure path: launches one CTA whose thread waits,
 * with the library's bounded wait, on an mbarrier that nothing completes.
 * After limit_ns (1 ms .. 1 s, CR_ERR_INVALID_ARG otherwise) the wait gives
 * up, sets the device error word exactly as a stalled pipeline would, and
 * the kernel returns; cr_check_device_error then reports CR_ERR_TIMEOUT and
 * clears the word.  No fault, trap or hang is involved and the context stays
 * usable.
 */
cr_status cr_selftest_wait_timeout(uint64_t limit_ns, cr_stream_t stream);

/*
 * (18) Measurement of the dense INT8 tensor-core rate (the prefill GEMM's
 * roofline denominator; not part of the layer).  Launches one cluster of two
 * CTAs per SM pair; each pair issues `iters` (1 .. 2^20) groups of four
 * tcgen05.mma.cta_group::2.kind::i8 (M = 256, N = 256, K = 32, the prefill
 * GEMM's instruction) on int8 tiles resident in shared memory, accumulating
 * in TMEM, with no global memory traffic.  *ops_per_launch (host) receives
 * the int8 operations one launch performs (2 * 256 * 256 * 128 * iters per
 * pair); the caller times the launch on `stream` (CUDA events) and divides.
 */
cr_status cr_mma_i8_peak(int64_t iters, double *ops_per_launch, cr_stream_t stream);

/*
 * Waits for `stream`, then reads and clears the library's device error word,
 * which a kernel sets when one of its bounded pipeline waits runs out (the
 * kernel then abandons its tile and exits; its outputs are unspecified).
 * Returns CR_OK, CR_ERR_TIMEOUT, or CR_ERR_CUDA if the wait itself failed.
 * This is the one synchronising call in the library.
 */
cr_status cr_check_device_error(cr_stream_t stream);

/* Library version, e.g. "0.1.0".  Host only. */
const char *cr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CR_W4A8_H */
