/*
 * cr_oracle.c -- plain, slow, scalar CPU oracle for the ConvRot W4A8 codebook
 * linear layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The CUDA library never
 * links, includes or calls it, and it shares no source with the CUDA library.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math -fPIC -shared
 * (oracle/build.py).  FP contraction is off so every float expression below
 * rounds exactly where it is written; x86-64 evaluates float in float
 * (FLT_EVAL_METHOD == 0) under the default round-to-nearest-even mode, and
 * subnormals are kept (no flush-to-zero).
 *
 * Sources (page title, then section):
 *   [CR]  ai-toolkit convrot_w4a8_quant.py -- module docstring (storage
 *         formula, buffers), FIXED_CODEBOOK, W4A8_SAT, _pack_codes /
 *         _unpack_codes, unpack_w4a8_eager, w4a8_gemv_kernel (int32
 *         multiply-accumulate and epilogue), w4a8_act_quant_kernel, _gemv_mp,
 *         _w4a8_linear_ste_op (unpack -> act quant -> _int_mm -> epilogue),
 *         dequantize_w4a8.
 *   [H3]  h3-rs src/weights.rs -- hadamard(), rotate_activation(),
 *         interleave_rows / QLinear::interleave_swiglu, swiglu_interleaved.
 *
 * Every function restates one definition.  Where the pages leave a detail
 * open (the fp32 summation order of the rotation, NaN handling, the
 * epilogue's multiply order) the reading taken is stated at the function.
 *
 * Parity status: every function here is pinned by a CPU test against the
 * pages' statements, closed forms, library routines or brute force
 * (tests/test_oracle_pins.py).  The quality of the quantised layer against
 * the unquantised weight is not a parity target and is not pinned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------
 * fp8 e4m3fn -> fp32.  [CR] w4a8_gemv_kernel and _fp8_rep8 reinterpret the
 * scale byte as float8e4nv.  e4m3fn: 1 sign bit, 4 exponent bits (bias 7),
 * 3 mantissa bits, no infinities, S.1111.111 is NaN.  Exact in fp32.
 * ------------------------------------------------------------------------ */
float or_fp8_e4m3fn_to_f32(uint8_t byte)
{
    int sign = (byte >> 7) & 1;
    int e = (byte >> 3) & 0xF;
    int m = byte & 0x7;
    double v;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);        /* subnormal: (m/8) * 2^(1-7) */
    else
        v = ldexp(1.0 + m / 8.0, e - 7); /* normal: (1 + m/8) * 2^(e-7) */
    return (float)(sign ? -v : v);
}

/* ------------------------------------------------------------------------
 * bf16 <-> fp32.  bf16 is the top half of an fp32, so widening is exact.
 * Narrowing rounds to nearest, ties to even.  NaN stays a quiet NaN.
 * ------------------------------------------------------------------------ */
float or_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

uint16_t or_f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if (isnan(f))
        return (uint16_t)(((u >> 16) & 0x8000u) | 0x7FC0u);
    /* Round the low 16 bits away: add 0x7FFF, plus 1 when the kept lsb is odd
     * (so an exact half goes to the even neighbour), then truncate. */
    uint32_t keep_lsb = (u >> 16) & 1u;
    u += 0x7FFFu + keep_lsb;
    return (uint16_t)(u >> 16);
}

/* double -> bf16 bits, one rounding to nearest, ties to even (used where the
 * oracle computes a value in double and the output is bf16, so that it is not
 * rounded twice through fp32).  Magnitudes below the smallest normal bf16 go
 * through fp32; NaN stays a quiet NaN; overflow gives an infinity. */
uint16_t or_f64_to_bf16_rne(double d)
{
    if (isnan(d))
        return (uint16_t)(signbit(d) ? 0xFFC0u : 0x7FC0u);
    if (fabs(d) < 1.1754943508222875e-38) /* 2^-126 */
        return or_f32_to_bf16_rne((float)d);
    uint64_t u;
    memcpy(&u, &d, 8);
    /* keep 7 of the 52 fraction bits: drop 45 with round-half-even */
    uint64_t keep_lsb = (u >> 45) & 1u;
    u += ((uint64_t)1 << 44) - 1 + keep_lsb;
    u &= ~(((uint64_t)1 << 45) - 1);
    double r;
    memcpy(&r, &u, 8);
    float f = (float)r; /* exact: 8 significant bits, in the fp32 exponent range, or an infinity */
    uint32_t b;
    memcpy(&b, &f, 4);
    return (uint16_t)(b >> 16);
}

/* ------------------------------------------------------------------------
 * Packed codes.  [CR] _pack_codes / _unpack_codes: byte j of a row holds
 * column 2j in its low nibble and column 2j+1 in its high nibble.
 * qdata [N, KH] bytes -> codes [N, 2*KH] (values 0..15).
 * ------------------------------------------------------------------------ */
void or_unpack_codes(const uint8_t *qdata, int64_t N, int64_t KH, uint8_t *codes)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < KH; ++j) {
            uint8_t b = qdata[n * KH + j];
            codes[n * 2 * KH + 2 * j] = b & 0xF;
            codes[n * 2 * KH + 2 * j + 1] = (b >> 4) & 0xF;
        }
}

/* ------------------------------------------------------------------------
 * One weight onto the int8 grid.  [CR] module docstring (storage formula),
 * unpack_w4a8_eager and W4A8_SAT = True: p = codebook[code] * s_rel in fp32,
 * then round to nearest even and saturate to [-128, 127] (the kernels' single
 * saturating round-to-nearest-even conversion).  The docstring's
 * clamp(-127, 127) is the W4A8_SAT = False variant, which the kernels do not
 * run.  Reading: a NaN product maps to 0, as that saturating conversion does.
 * ------------------------------------------------------------------------ */
int8_t or_decode_one(float cb_value, float srel_value)
{
    float p = cb_value * srel_value;
    if (isnan(p))
        return 0;
    float r = rintf(p); /* default rounding mode: nearest, ties to even */
    if (r < -128.0f)
        r = -128.0f;
    if (r > 127.0f)
        r = 127.0f;
    return (int8_t)r;
}

/* [CR] unpack_w4a8_eager with group size 16: qdata [N, K/2] packed codes,
 * srel [N, K/16] fp8 e4m3fn bytes, codebook[16] fp32 -> w8 [N, K] int8. */
void or_decode_w8(const uint8_t *qdata, const uint8_t *srel, const float *codebook,
                  int64_t N, int64_t K, int8_t *w8)
{
    const int64_t KH = K / 2, KG = K / 16;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t b = qdata[n * KH + k / 2];
            int code = (k % 2 == 0) ? (b & 0xF) : ((b >> 4) & 0xF);
            float s = or_fp8_e4m3fn_to_f32(srel[n * KG + k / 16]);
            w8[n * K + k] = or_decode_one(codebook[code], s);
        }
}

/* ------------------------------------------------------------------------
 * Dense regular Hadamard.  [H3] hadamard(): start from the 4x4 regular
 * Hadamard h4 (all ones except -1 on the anti-diagonal); each step replaces
 * H_n by H_4n with H_4n[4i+a][4j+b] = H_n[i][j] * h4[a][b]; stop at `size`
 * (which must be a power of 4) and divide every entry by sqrt(size).
 * Built in fp64.  Returns 0, or -1 if size is not a power of 4.
 * ------------------------------------------------------------------------ */
static const double OR_H4[4][4] = {
    {1, 1, 1, -1},
    {1, 1, -1, 1},
    {1, -1, 1, 1},
    {-1, 1, 1, 1},
};

int or_hadamard_dense(int size, double *H /* [size][size], row-major */)
{
    int n = 4;
    int p = 4;
    while (p < size)
        p *= 4;
    if (p != size)
        return -1; /* not a power of 4 (the page bails out the same way) */
    double *cur = (double *)malloc(sizeof(double) * (size_t)size * (size_t)size);
    double *nxt = (double *)malloc(sizeof(double) * (size_t)size * (size_t)size);
    if (!cur || !nxt) {
        free(cur);
        free(nxt);
        return -2;
    }
    for (int a = 0; a < 4; ++a)
        for (int b = 0; b < 4; ++b)
            cur[a * 4 + b] = OR_H4[a][b];
    while (n < size) {
        int n4 = 4 * n;
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j)
                for (int a = 0; a < 4; ++a)
                    for (int b = 0; b < 4; ++b)
                        nxt[(int64_t)(4 * i + a) * n4 + (4 * j + b)] =
                            cur[(int64_t)i * n + j] * OR_H4[a][b];
        double *t = cur;
        cur = nxt;
        nxt = t;
        n = n4;
    }
    if (n != size) {
        free(cur);
        free(nxt);
        return -1;
    }
    double norm = sqrt((double)size);
    for (int64_t i = 0; i < (int64_t)size * size; ++i)
        H[i] = cur[i] / norm;
    free(cur);
    free(nxt);
    return 0;
}

/* ------------------------------------------------------------------------
 * Block-256 rotation of one activation row, in fp32.
 *
 * Definition: r[b*256 : (b+1)*256] = x[b*256 : (b+1)*256] @ H_256 with
 * H_256 = (h4 (x) h4 (x) h4 (x) h4) / 16 ([H3] hadamard, rotate_activation:
 * the row is cut into blocks of the rotation size and each block is
 * multiplied by H).  Because H_256 is a Kronecker power, x @ H_256 applies
 * h4 along each base-4 digit of the index within the block (index
 * i = 64*d3 + 16*d2 + 4*d1 + d0).
 *
 * Reading (the pages fix neither the precision nor the order of the fp32
 * sums): the bf16 inputs are widened exactly to fp32 and never rounded to
 * bf16 again.  The digits are processed in the order d0, d1, d2, d3 (index
 * strides 1, 4, 16, 64).  For one quadruple (v0, v1, v2, v3) along a digit,
 * output a is  S - 2*v[3-a]  with  S = (v0 + v1) + (v2 + v3),  which equals
 * sum_b h4[a][b]*v[b] because row a of h4 is all ones except -1 at column
 * 3-a.  2*v is exact, so S - 2*v rounds once.  After the four digits every
 * value is multiplied by 1/16 (exact unless the result is subnormal).
 * ------------------------------------------------------------------------ */
static void or_rotate_block256(float *v /* 256 values, in place */)
{
    static const int strides[4] = {1, 4, 16, 64};
    for (int t = 0; t < 4; ++t) {
        int s = strides[t];
        for (int i = 0; i < 256; ++i) {
            if ((i / s) % 4 != 0)
                continue; /* i is the first element of its quadruple */
            float q[4] = {v[i], v[i + s], v[i + 2 * s], v[i + 3 * s]};
            float S = (q[0] + q[1]) + (q[2] + q[3]);
            for (int a = 0; a < 4; ++a) {
                float twice = 2.0f * q[3 - a];
                v[i + a * s] = S - twice;
            }
        }
    }
    for (int i = 0; i < 256; ++i)
        v[i] = v[i] * 0.0625f;
}

/* x [M, K] bf16 bits -> r [M, K] fp32 rotated.  K must be a multiple of 256.
 * Returns 0, or -1 on a bad K. */
int or_rotate_rows(const uint16_t *x, int64_t M, int64_t K, float *r)
{
    if (K <= 0 || K % 256 != 0)
        return -1;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t b = 0; b < K / 256; ++b) {
            float *blk = r + m * K + b * 256;
            for (int i = 0; i < 256; ++i)
                blk[i] = or_bf16_to_f32(x[m * K + b * 256 + i]);
            or_rotate_block256(blk);
        }
    return 0;
}

/* ------------------------------------------------------------------------
 * Per-token symmetric int8 quantisation.  [CR] w4a8_act_quant_kernel:
 *   amax  = max_k |r[m,k]|               (exact under any order)
 *   scale = amax > 0 ? amax / qmax : 1   (fp32 division)
 *   q     = clamp(rint(r / scale), -qmax, qmax)
 * into exactly MP rows: rows m >= M get q = 0 and scale = 1 ([CR] "rows >= M:
 * zeros, scale 1").  Reading: the prefill quantiser (_int8_act_quant_padded,
 * not on the pages) is the same arithmetic, which the pages state when they
 * call the decode GEMV bit-identical to the _int_mm path.  qmax is the
 * module's act_qmax; the default reading is 127.
 *
 * The max follows C fmaxf (a NaN operand is ignored); the activations are
 * expected finite, and no further NaN rule is defined.
 * ------------------------------------------------------------------------ */
int or_act_quant_rows(const float *r, int64_t M, int64_t K, int64_t MP, int qmax,
                      int8_t *xq, float *xs)
{
    if (MP < M || qmax < 1 || qmax > 127)
        return -1;
    for (int64_t m = 0; m < MP; ++m) {
        if (m >= M) {
            for (int64_t k = 0; k < K; ++k)
                xq[m * K + k] = 0;
            xs[m] = 1.0f;
            continue;
        }
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k)
            amax = fmaxf(amax, fabsf(r[m * K + k]));
        float scale = (amax > 0.0f) ? amax / (float)qmax : 1.0f;
        for (int64_t k = 0; k < K; ++k) {
            float q = rintf(r[m * K + k] / scale);
            if (q < (float)-qmax)
                q = (float)-qmax;
            if (q > (float)qmax)
                q = (float)qmax;
            xq[m * K + k] = (int8_t)q;
        }
        xs[m] = scale;
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * int8 x int8 -> int32 contraction.  [CR] _w4a8_linear_ste_op
 * (torch._int_mm(aq, w8.t())) and w4a8_gemv_kernel (int32 multiply-
 * accumulate, exact and order independent):
 *   acc[m, n] = sum_k xq[m, k] * w8[n, k].
 * Summed in int64; returns -1 if any result leaves the int32 range (it cannot
 * for |xq| <= 127, |w8| <= 128 and K <= 132104).  Rows [m0, m1) only, so a
 * caller may split the work.
 * ------------------------------------------------------------------------ */
int or_gemm_s32_rows(const int8_t *xq, const int8_t *w8, int64_t m0, int64_t m1,
                     int64_t N, int64_t K, int32_t *acc /* [M, N], rows m0..m1 */)
{
    int bad = 0;
    for (int64_t m = m0; m < m1; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k)
                s += (int64_t)xq[m * K + k] * (int64_t)w8[n * K + k];
            if (s > INT32_MAX || s < INT32_MIN)
                bad = 1;
            acc[m * N + n] = (int32_t)s;
        }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------
 * Epilogue.  [CR] w4a8_gemv_kernel epilogue: out = float(acc) * (xs[m] *
 * ws[n]) (+ bias[n]), then cast to the output dtype.  Reading: exactly that
 * parenthesisation, each operation rounded on its own (no fused multiply-add),
 * bias added last; the prefill epilogue (_int8_epilogue, not on the pages) is
 * the same formula, since the pages call the two paths bit-identical.
 * out_bf16 != 0: out is bf16 bits [M, N] (round to nearest even); else fp32.
 * bias may be NULL.
 * ------------------------------------------------------------------------ */
void or_epilogue(const int32_t *acc, const float *xs, const float *ws, const float *bias,
                 int64_t M, int64_t N, int out_bf16, void *out)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            float t = (float)acc[m * N + n]; /* int32 -> fp32, nearest even */
            float sc = xs[m] * ws[n];
            float y = t * sc;
            if (bias)
                y = y + bias[n];
            if (out_bf16)
                ((uint16_t *)out)[m * N + n] = or_f32_to_bf16_rne(y);
            else
                ((float *)out)[m * N + n] = y;
        }
}

/* ------------------------------------------------------------------------
 * SwiGLU on row-interleaved gate/up outputs.  [H3] QLinear::interleave_swiglu
 * (a gate/up layer's output rows reordered to pairs g0, u0, g1, u1, ...) and
 * swiglu_interleaved (silu(gate) * up of each pair).
 * acc [M, 2F] int32.  g = the epilogue value of column 2f and u = that of
 * column 2f + 1, each in fp32 exactly as or_epilogue computes it (the pages'
 * fp32 rescale); then silu(g) * u = g * u / (1 + exp(-g)), which the pages
 * do not pin to a precision: here in double, rounded once to the output
 * type.  out [M, F].
 * ------------------------------------------------------------------------ */
void or_epilogue_swiglu(const int32_t *acc, const float *xs, const float *ws, const float *bias,
                        int64_t M, int64_t F, int out_bf16, void *out)
{
    const int64_t N = 2 * F;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t f = 0; f < F; ++f) {
            float v[2];
            for (int h = 0; h < 2; ++h) {
                const int64_t n = 2 * f + h;
                float t = (float)acc[m * N + n];
                float sc = xs[m] * ws[n];
                v[h] = t * sc;
                if (bias)
                    v[h] = v[h] + bias[n];
            }
            const double g = v[0], up = v[1];
            const double y = g / (1.0 + exp(-g)) * up;
            if (out_bf16)
                ((uint16_t *)out)[m * F + f] = or_f64_to_bf16_rne(y);
            else
                ((float *)out)[m * F + f] = (float)y;
        }
}

/* ========================================================================
 * Offline quantiser.  [CR] quantize_w4a8_rotated / _quantize_rotated_rows,
 * _assign_codes, _assign_grid, grid_levels, _ALS_ITERS = 2.
 * ======================================================================== */

/* fp32 -> fp8 e4m3fn byte, as torch's .to(torch.float8_e4m3fn) does (the
 * quantiser's s_rel cast): the value rounded to the nearest e4m3 number,
 * ties to even, where the pattern S.1111.111 (which would be 480) is NaN, so
 * a magnitude that rounds above 448 becomes NaN; no saturation.  Subnormals
 * (steps of 2^-9 below 2^-6) are kept; NaN and infinities give NaN. */
uint8_t or_f32_to_fp8_e4m3fn(float f)
{
    const uint8_t sign = signbit(f) ? 0x80 : 0x00;
    if (isnan(f) || isinf(f))
        return (uint8_t)(sign | 0x7F);
    double a = fabs((double)f);
    /* the grid step at a's binade: 2^(e-3) for normals, 2^-9 below 2^-6 */
    int e;
    frexp(a, &e); /* a = m * 2^e, m in [0.5, 1): the binade is [2^(e-1), 2^e) */
    int exp2 = e - 1;
    if (exp2 < -6)
        exp2 = -6;
    const double step = ldexp(1.0, exp2 - 3);
    double units = a / step; /* exact: a power-of-two division */
    double r = nearbyint(units); /* the default rounding mode: to nearest, ties to even */
    const double v = r * step;
    if (v >= 480.0)
        return (uint8_t)(sign | 0x7F);
    /* encode v (a multiple of step) */
    uint8_t code;
    if (v < ldexp(1.0, -6)) {
        code = (uint8_t)(v / ldexp(1.0, -9)); /* 0..8; 8 is 2^-6, the smallest normal */
    } else {
        int ev;
        const double m = frexp(v, &ev); /* v = m 2^ev, m in [0.5, 1) */
        const int ebias = ev - 1 + 7;
        const int mant = (int)((m * 2.0 - 1.0) * 8.0);
        code = (uint8_t)((ebias << 3) | mant);
    }
    return (uint8_t)(sign | code);
}

/* Count of the n non-decreasing levels strictly below x, i.e.
 * torch.searchsorted(levels, x) (left side) on a sorted row. */
static int or_searchsorted_left(const float *levels, int n, float x)
{
    int pos = 0;
    while (pos < n && levels[pos] < x)
        ++pos;
    return pos;
}

/* [CR] _assign_codes / deterministic _assign_grid: the bracketing pair of the
 * search position, each distance |x - level| in fp32, the upper level only
 * when strictly nearer (ties go to the lower index). */
int or_nearest_level(const float *levels, int n, float x)
{
    const int last = n - 1;
    const int pos = or_searchsorted_left(levels, n, x);
    const int lo = pos - 1 < 0 ? 0 : (pos - 1 > last ? last : pos - 1);
    const int hi = pos > last ? last : pos;
    const float dlo = fabsf(x - levels[lo]);
    const float dhi = fabsf(x - levels[hi]);
    return dhi < dlo ? hi : lo;
}

/* [CR] stochastic _assign_grid: lo = clamp(pos - 1, 0, n - 2), the threshold
 * u * (levels[lo + 1] - levels[lo]) + levels[lo] (a multiply, then an add,
 * each rounded to fp32), and the upper level when x is strictly above it.
 * u is the uniform [0, 1) draw for this weight (an input). */
int or_stochastic_level(const float *levels, int n, float x, float u)
{
    const int last = n - 1;
    const int pos = or_searchsorted_left(levels, n, x);
    int lo = pos - 1;
    if (lo < 0)
        lo = 0;
    if (lo > last - 1)
        lo = last - 1;
    const float level_lo = levels[lo];
    const float width = levels[lo + 1] - level_lo;
    const float uw = u * width;
    const float thr = uw + level_lo;
    int code = lo + (x > thr ? 1 : 0);
    return code > last ? last : code;
}

/* [CR] grid_levels: the int8 value each of the 16 codebook levels decodes to
 * for one fp8 group scale, round(codebook[i] * s_rel) (one fp32 multiply,
 * round half to even) clamped to [-127, 127]. */
void or_grid_levels(const float *codebook, uint8_t srel_byte, float *levels /* [16] */)
{
    const float s = or_fp8_e4m3fn_to_f32(srel_byte);
    for (int i = 0; i < 16; ++i) {
        float v = nearbyintf(codebook[i] * s);
        if (v < -127.0f)
            v = -127.0f;
        if (v > 127.0f)
            v = 127.0f;
        levels[i] = v;
    }
}

/* Sum of 16 fp32 values in a fixed pairwise order: ((v0+v1)+(v2+v3)) + ...,
 * then pairs of those, down to one.  The pages sum a group's 16 products with
 * torch's .sum(-1), whose order they do not fix; this order is the reading
 * taken (the GPU follows it exactly). */
static float or_sum16_pairwise(const float *v)
{
    float a[8], b[4], c[2];
    for (int i = 0; i < 8; ++i)
        a[i] = v[2 * i] + v[2 * i + 1];
    for (int i = 0; i < 4; ++i)
        b[i] = a[2 * i] + a[2 * i + 1];
    for (int i = 0; i < 2; ++i)
        c[i] = b[2 * i] + b[2 * i + 1];
    return c[0] + c[1];
}

static float or_clamp_min(float v, float lo)
{
    return v < lo ? lo : v; /* torch clamp(min=lo): NaN stays NaN */
}

/* Per group of 16 rotated weights gw: the group scale after the ALS passes
 * ([CR] _quantize_rotated_rows): gs = clamp(max|gw|, 1e-8); codes = nearest
 * codebook index of gw / gs; then _ALS_ITERS = 2 times: lv = codebook[codes],
 * gs = clamp(sum(gw * lv) / clamp(sum(lv * lv), 1e-8), 1e-8), codes = nearest
 * index of gw / gs.  Writes the final codes of this stage to q. */
float or_group_scale_als(const float *gw, const float *codebook, int *q /* [16] */)
{
    const float eps = 1e-8f;
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        const float a = fabsf(gw[i]);
        if (a > amax)
            amax = a;
    }
    float gs = or_clamp_min(amax, eps);
    for (int i = 0; i < 16; ++i)
        q[i] = or_nearest_level(codebook, 16, gw[i] / gs);
    for (int it = 0; it < 2; ++it) {
        float p[16], l2[16];
        for (int i = 0; i < 16; ++i) {
            const float lv = codebook[q[i]];
            p[i] = gw[i] * lv;
            l2[i] = lv * lv;
        }
        const float num = or_sum16_pairwise(p);
        const float den = or_clamp_min(or_sum16_pairwise(l2), eps);
        gs = or_clamp_min(num / den, eps);
        for (int i = 0; i < 16; ++i)
            q[i] = or_nearest_level(codebook, 16, gw[i] / gs);
    }
    return gs;
}

/* [CR] _assign_grid on one group of 16 rotated weights: target = w / s_channel
 * (an fp32 division), then the nearest level of the group's grid, or with
 * rand != NULL the stochastic choice with rand[i] as the draw of weight i.
 * The quantiser's final assignment and the code re-assignment both run it,
 * as the page's _quantize_rotated_rows and requantize_codes_ (and
 * fake_quant_rotated_weight) all call _assign_grid on w / s_channel and
 * grid_levels(codebook, s_rel). */
static void or_assign_group(const float *w, float s_channel, const float *levels, const float *rand, int *c)
{
    for (int i = 0; i < 16; ++i) {
        const float t = w[i] / s_channel;
        c[i] = rand ? or_stochastic_level(levels, 16, t, rand[i]) : or_nearest_level(levels, 16, t);
    }
}

/* [CR] quantize_w4a8_rotated (row chunking does not change the result: rows
 * are independent).  w_rot [N, K] fp32 (already rotated), K a multiple of 16.
 * Per row: the group scales gs and codes of or_group_scale_als; s_channel =
 * clamp(max |codebook[code] * gs| / 127, 1e-8); s_rel = fp8(gs / s_channel);
 * final codes = nearest level of w_rot / s_channel on grid_levels(s_rel);
 * packed with column 2j in the low nibble of byte j.
 * Outputs: qdata [N, K/2], srel [N, K/16] fp8 bytes, s_channel [N]. */
int or_quantize_rotated(const float *w_rot, int64_t N, int64_t K, const float *codebook, uint8_t *qdata,
                        uint8_t *srel, float *s_channel)
{
    if (K % 16 != 0 || N < 0 || K < 0)
        return -1;
    const int64_t G = K / 16;
    float *gs = (float *)malloc((size_t)(G > 0 ? G : 1) * sizeof(float));
    if (!gs)
        return -1;
    for (int64_t n = 0; n < N; ++n) {
        const float *row = w_rot + n * K;
        float rowmax = 0.0f;
        for (int64_t g = 0; g < G; ++g) {
            int q[16];
            gs[g] = or_group_scale_als(row + 16 * g, codebook, q);
            for (int i = 0; i < 16; ++i) {
                const float a = fabsf(codebook[q[i]] * gs[g]);
                if (a > rowmax)
                    rowmax = a;
            }
        }
        const float sch = or_clamp_min(rowmax / 127.0f, 1e-8f);
        s_channel[n] = sch;
        for (int64_t g = 0; g < G; ++g) {
            const uint8_t b = or_f32_to_fp8_e4m3fn(gs[g] / sch);
            srel[n * G + g] = b;
            float levels[16];
            or_grid_levels(codebook, b, levels);
            int c[16];
            or_assign_group(row + 16 * g, sch, levels, NULL, c);
            for (int i = 0; i < 16; i += 2)
                qdata[n * (K / 2) + 8 * g + i / 2] = (uint8_t)(c[i] | (c[i + 1] << 4));
        }
    }
    free(gs);
    return 0;
}

/* [CR] requantize_codes_ without its rotation: new codes for rotated weights
 * on STORED scales.  target = w_rot / s_channel; levels = grid_levels(s_rel);
 * deterministic nearest level, or (rand != NULL) the stochastic choice with
 * rand[n, k] as the uniform draw of weight (n, k).  Output packed qdata. */
int or_assign_codes(const float *w_rot, const uint8_t *srel, const float *s_channel, const float *codebook,
                    const float *rand, int64_t N, int64_t K, uint8_t *qdata)
{
    if (K % 16 != 0 || N < 0 || K < 0)
        return -1;
    const int64_t G = K / 16;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < G; ++g) {
            float levels[16];
            or_grid_levels(codebook, srel[n * G + g], levels);
            int c[16];
            or_assign_group(w_rot + n * K + 16 * g, s_channel[n], levels, rand ? rand + n * K + 16 * g : NULL, c);
            for (int i = 0; i < 16; i += 2)
                qdata[n * (K / 2) + 8 * g + i / 2] = (uint8_t)(c[i] | (c[i + 1] << 4));
        }
    return 0;
}

/* ========================================================================
 * Straight-through backward.  [CR] _w4a8_linear_ste_backward: the codes are
 * decoded again, w = w8.to(grad.dtype) * s_channel.to(grad.dtype), and the
 * input gradient is grad @ w.
 * ======================================================================== */

/* The dequantised weight in bf16, as the backward builds it for bf16
 * gradients: w8 (exact in bf16) times bf16(s_channel[n]), the product of two
 * bf16 values (exact in fp32) rounded once to bf16.  w [N, K] bf16 bits. */
void or_dequant_bf16(const uint8_t *qdata, const uint8_t *srel, const float *codebook, const float *s_channel,
                     int64_t N, int64_t K, uint16_t *w)
{
    int8_t *w8 = (int8_t *)malloc((size_t)(N * K > 0 ? N * K : 1));
    if (!w8)
        return;
    or_decode_w8(qdata, srel, codebook, N, K, w8);
    for (int64_t n = 0; n < N; ++n) {
        const float s = or_bf16_to_f32(or_f32_to_bf16_rne(s_channel[n]));
        for (int64_t k = 0; k < K; ++k)
            w[n * K + k] = or_f32_to_bf16_rne((float)w8[n * K + k] * s);
    }
    free(w8);
}

/* dx [M, K] bf16 = grad [M, N] bf16 @ w [N, K] bf16 (or_dequant_bf16).  The
 * pages leave the accumulation to the matmul; here every product and sum is
 * in double and the result is rounded once to bf16. */
int or_ste_backward(const uint16_t *grad, const uint8_t *qdata, const uint8_t *srel, const float *codebook,
                    const float *s_channel, int64_t M, int64_t N, int64_t K, uint16_t *dx)
{
    uint16_t *w = (uint16_t *)malloc((size_t)(N * K > 0 ? N * K : 1) * sizeof(uint16_t));
    double *row = (double *)malloc((size_t)(K > 0 ? K : 1) * sizeof(double));
    if (!w || !row) {
        free(w);
        free(row);
        return -1;
    }
    or_dequant_bf16(qdata, srel, codebook, s_channel, N, K, w);
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k)
            row[k] = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            const double g = or_bf16_to_f32(grad[m * N + n]);
            if (g == 0.0)
                continue;
            const uint16_t *wr = w + n * K;
            for (int64_t k = 0; k < K; ++k)
                row[k] += g * (double)or_bf16_to_f32(wr[k]);
        }
        for (int64_t k = 0; k < K; ++k)
            dx[m * K + k] = or_f64_to_bf16_rne(row[k]);
    }
    free(w);
    free(row);
    return 0;
}
