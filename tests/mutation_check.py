"""Mutation check of the oracle's CPU pins.

Each entry below is a plausible mistake in the oracle (a wrong rounding, a
swapped operand, a dropped step, another order of operations).  The script
applies one at a time to a copy of oracle/ in a work directory, rebuilds the
copy and runs tests/test_oracle_pins.py against it; every mutation must make
at least one pin fail, except the few listed in EQUIVALENT, which change no
result on any input the oracle accepts (the reason is given with each).

    python tests/mutation_check.py --work <scratch dir> [name ...]

It is not collected by pytest (about a minute and a half on 6 workers).
"""
import argparse
import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
C = "oracle/cr_oracle.c"

MUTATIONS = [
 ("fp8_sub_scale", C, "v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
 ("fp8_nan_rule", C, "if (e == 0xF && m == 0x7)\n        return NAN;", "if (e == 0xF)\n        return NAN;"),
 ("fp8_bias", C, "v = ldexp(1.0 + m / 8.0, e - 7);", "v = ldexp(1.0 + m / 8.0, e - 8);"),
 ("bf16_half_up", C, "u += 0x7FFFu + keep_lsb;", "u += 0x8000u;"),
 ("bf16_trunc", C, "u += 0x7FFFu + keep_lsb;", "u += 0u;"),
 ("f64bf16_half_up", C, "u += ((uint64_t)1 << 44) - 1 + keep_lsb;", "u += ((uint64_t)1 << 44);"),
 ("f64bf16_via_f32", C, "    if (fabs(d) < 1.1754943508222875e-38) /* 2^-126 */\n        return or_f32_to_bf16_rne((float)d);", "    return or_f32_to_bf16_rne((float)d);"),
 ("unpack_swap", C, "codes[n * 2 * KH + 2 * j] = b & 0xF;\n            codes[n * 2 * KH + 2 * j + 1] = (b >> 4) & 0xF;", "codes[n * 2 * KH + 2 * j] = (b >> 4) & 0xF;\n            codes[n * 2 * KH + 2 * j + 1] = b & 0xF;"),
 ("decode_roundaway", C, "float r = rintf(p); /* default", "float r = roundf(p); /* default"),
 ("decode_sat127", C, "if (r < -128.0f)\n        r = -128.0f;", "if (r < -127.0f)\n        r = -127.0f;"),
 ("decode_nan_m128", C, "if (isnan(p))\n        return 0;", "if (isnan(p))\n        return -128;"),
 ("decode_double", C, "    float p = cb_value * srel_value;\n    if (isnan(p))\n        return 0;\n    float r = rintf(p);", "    double p = (double)cb_value * srel_value;\n    if (isnan(p))\n        return 0;\n    float r = (float)rint(p);"),
 ("decode_w8_nibble", C, "int code = (k % 2 == 0) ? (b & 0xF) : ((b >> 4) & 0xF);", "int code = (k % 2 == 1) ? (b & 0xF) : ((b >> 4) & 0xF);"),
 ("decode_w8_group32", C, "float s = or_fp8_e4m3fn_to_f32(srel[n * KG + k / 16]);", "float s = or_fp8_e4m3fn_to_f32(srel[n * KG + k / 32]);"),
 ("h4_rows_swapped", C, "    {1, 1, 1, -1},\n    {1, 1, -1, 1},\n    {1, -1, 1, 1},\n    {-1, 1, 1, 1},", "    {-1, 1, 1, 1},\n    {1, 1, -1, 1},\n    {1, -1, 1, 1},\n    {1, 1, 1, -1},"),
 ("had_norm", C, "double norm = sqrt((double)size);", "double norm = (double)size;"),
 ("rot_order_rev", C, "static const int strides[4] = {1, 4, 16, 64};", "static const int strides[4] = {64, 16, 4, 1};"),
 ("rot_order_swap12", C, "static const int strides[4] = {1, 4, 16, 64};", "static const int strides[4] = {1, 16, 4, 64};"),
 ("rot_diag", C, "float twice = 2.0f * q[3 - a];", "float twice = 2.0f * q[a];"),
 ("rot_seq_sum", C, "float S = (q[0] + q[1]) + (q[2] + q[3]);", "float S = ((q[0] + q[1]) + q[2]) + q[3];"),
 ("rot_sum_pairs02", C, "float S = (q[0] + q[1]) + (q[2] + q[3]);", "float S = (q[0] + q[2]) + (q[1] + q[3]);"),
 ("rot_scale", C, "v[i] = v[i] * 0.0625f;", "v[i] = v[i] * 0.125f;"),
 ("rot_scale_first", C, "                float twice = 2.0f * q[3 - a];\n                v[i + a * s] = S - twice;", "                float twice = 2.0f * q[3 - a];\n                v[i + a * s] = (S - twice) * (t == 0 ? 0.0625f : 1.0f);"),
 ("aq_noabs", C, "amax = fmaxf(amax, fabsf(r[m * K + k]));", "amax = fmaxf(amax, r[m * K + k]);"),
 ("aq_recip", C, "float scale = (amax > 0.0f) ? amax / (float)qmax : 1.0f;", "float scale = (amax > 0.0f) ? amax * (1.0f / (float)qmax) : 1.0f;"),
 ("aq_mulrecip", C, "float q = rintf(r[m * K + k] / scale);", "float q = rintf(r[m * K + k] * (1.0f / scale));"),
 ("aq_roundaway", C, "float q = rintf(r[m * K + k] / scale);", "float q = roundf(r[m * K + k] / scale);"),
 ("aq_clamp", C, "if (q < (float)-qmax)\n                q = (float)-qmax;", "if (q < (float)(-qmax - 1))\n                q = (float)(-qmax - 1);"),
 ("aq_pad_scale0", C, "xs[m] = 1.0f;\n            continue;", "xs[m] = 0.0f;\n            continue;"),
 ("aq_zero_scale", C, "float scale = (amax > 0.0f) ? amax / (float)qmax : 1.0f;", "float scale = (amax > 0.0f) ? amax / (float)qmax : 0.0f;"),
 ("gemm_wrap", C, "if (s > INT32_MAX || s < INT32_MIN)\n                bad = 1;", "(void)0;"),
 ("epi_order", C, "float sc = xs[m] * ws[n];\n            float y = t * sc;", "float y = (t * xs[m]) * ws[n];"),
 ("epi_bias_first", C, "            float y = t * sc;\n            if (bias)\n                y = y + bias[n];", "            float y = t;\n            if (bias)\n                y = (y + bias[n] / sc);\n            y = y * sc;"),
 ("epi_fma", C, "            float y = t * sc;\n            if (bias)\n                y = y + bias[n];", "            float y = t * sc;\n            if (bias)\n                y = fmaf(t, sc, bias[n]);"),
 ("swi_sign", C, "const double y = g / (1.0 + exp(-g)) * up;", "const double y = g / (1.0 + exp(g)) * up;"),
 ("swi_swap", C, "const double g = v[0], up = v[1];", "const double g = v[1], up = v[0];"),
 ("swi_f32", C, "const double y = g / (1.0 + exp(-g)) * up;", "const double y = (float)((float)(g / (1.0 + exp(-g))) * (float)up);"),
 ("fp8enc_away", C, "double r = nearbyint(units);", "double r = round(units);"),
 ("fp8enc_sat", C, "    if (v >= 480.0)\n        return (uint8_t)(sign | 0x7F);", "    if (v >= 480.0)\n        return (uint8_t)(sign | 0x7E);"),
 ("fp8enc_sub", C, "    if (exp2 < -6)\n        exp2 = -6;", "    if (exp2 < -7)\n        exp2 = -7;"),
 ("fp8enc_inf_sat", C, "    if (isnan(f) || isinf(f))\n        return (uint8_t)(sign | 0x7F);", "    if (isnan(f))\n        return (uint8_t)(sign | 0x7F);\n    if (isinf(f))\n        return (uint8_t)(sign | 0x7E);"),
 ("ss_right", C, "while (pos < n && levels[pos] < x)", "while (pos < n && levels[pos] <= x)"),
 ("near_tie_up", C, "return dhi < dlo ? hi : lo;", "return dhi <= dlo ? hi : lo;"),
 ("stoch_ge", C, "int code = lo + (x > thr ? 1 : 0);", "int code = lo + (x >= thr ? 1 : 0);"),
 ("stoch_1mu", C, "const float uw = u * width;", "const float uw = (1.0f - u) * width;"),
 ("stoch_fma", C, "const float uw = u * width;\n    const float thr = uw + level_lo;", "const float thr = fmaf(u, width, level_lo);"),
 ("stoch_lo_clamp", C, "    if (lo > last - 1)\n        lo = last - 1;", "    if (lo > last)\n        lo = last;"),
 ("grid_clamp128", C, "        if (v < -127.0f)\n            v = -127.0f;", "        if (v < -128.0f)\n            v = -128.0f;"),
 ("grid_roundaway", C, "float v = nearbyintf(codebook[i] * s);", "float v = roundf(codebook[i] * s);"),
 ("sum16_seq", C, "static float or_sum16_pairwise(const float *v)\n{", "static float or_sum16_pairwise(const float *v)\n{\n    if (1) { float s = 0.0f; for (int i = 0; i < 16; ++i) s += v[i]; return s; }"),
 ("als_once", C, "for (int it = 0; it < 2; ++it) {", "for (int it = 0; it < 1; ++it) {"),
 ("als_thrice", C, "for (int it = 0; it < 2; ++it) {", "for (int it = 0; it < 3; ++it) {"),
 ("als_eps", C, "const float eps = 1e-8f;", "const float eps = 1e-6f;"),
 ("als_no_requant", C, "        gs = or_clamp_min(num / den, eps);\n        for (int i = 0; i < 16; ++i)\n            q[i] = or_nearest_level(codebook, 16, gw[i] / gs);", "        gs = or_clamp_min(num / den, eps);"),
 ("q_rowmax_gs", C, "const float a = fabsf(codebook[q[i]] * gs[g]);", "const float a = fabsf(gs[g]);"),
 ("q_div128", C, "const float sch = or_clamp_min(rowmax / 127.0f, 1e-8f);", "const float sch = or_clamp_min(rowmax / 128.0f, 1e-8f);"),
 ("q_pack_swap", C, "            or_assign_group(row + 16 * g, sch, levels, NULL, c);\n            for (int i = 0; i < 16; i += 2)\n                qdata[n * (K / 2) + 8 * g + i / 2] = (uint8_t)(c[i] | (c[i + 1] << 4));", "            or_assign_group(row + 16 * g, sch, levels, NULL, c);\n            for (int i = 0; i < 16; i += 2)\n                qdata[n * (K / 2) + 8 * g + i / 2] = (uint8_t)(c[i + 1] | (c[i] << 4));"),
 ("assign_mul", C, "const float t = w[i] / s_channel;", "const float t = w[i] * (1.0f / s_channel);"),
 ("q_final_direct", C, "            or_assign_group(row + 16 * g, sch, levels, NULL, c);", "            for (int i = 0; i < 16; ++i) c[i] = or_nearest_level(levels, 16, row[16 * g + i] * (1.0f / sch));"),
 ("als_recip", C, "        for (int i = 0; i < 16; ++i)\n            q[i] = or_nearest_level(codebook, 16, gw[i] / gs);\n    }", "        for (int i = 0; i < 16; ++i)\n            q[i] = or_nearest_level(codebook, 16, gw[i] * (1.0f / gs));\n    }"),
 ("als_recip0", C, "    float gs = or_clamp_min(amax, eps);\n    for (int i = 0; i < 16; ++i)\n        q[i] = or_nearest_level(codebook, 16, gw[i] / gs);", "    float gs = or_clamp_min(amax, eps);\n    for (int i = 0; i < 16; ++i)\n        q[i] = or_nearest_level(codebook, 16, gw[i] * (1.0f / gs));"),
 ("als_quot_recip", C, "gs = or_clamp_min(num / den, eps);", "gs = or_clamp_min(num * (1.0f / den), eps);"),
 ("q_srel_recip", C, "const uint8_t b = or_f32_to_fp8_e4m3fn(gs[g] / sch);", "const uint8_t b = or_f32_to_fp8_e4m3fn(gs[g] * (1.0f / sch));"),
 ("q_sch_recip", C, "const float sch = or_clamp_min(rowmax / 127.0f, 1e-8f);", "const float sch = or_clamp_min(rowmax * (1.0f / 127.0f), 1e-8f);"),
 ("q_sch_floor", C, "const float sch = or_clamp_min(rowmax / 127.0f, 1e-8f);", "const float sch = or_clamp_min(rowmax / 127.0f, 1e-9f);"),
 ("als_den_floor", C, "const float den = or_clamp_min(or_sum16_pairwise(l2), eps);", "const float den = or_sum16_pairwise(l2);"),
 ("epi_i2f_trunc", C, "float t = (float)acc[m * N + n]; /* int32 -> fp32, nearest even */", "float t = (float)(double)(acc[m * N + n] & ~0xFF);"),
 ("swi_bias_in", C, "                v[h] = t * sc;\n                if (bias)\n                    v[h] = v[h] + bias[n];", "                v[h] = t * sc;"),
 ("assign_pack_swap", C, "rand ? rand + n * K + 16 * g : NULL, c);\n            for (int i = 0; i < 16; i += 2)\n                qdata[n * (K / 2) + 8 * g + i / 2] = (uint8_t)(c[i] | (c[i + 1] << 4));", "rand ? rand + n * K + 16 * g : NULL, c);\n            for (int i = 0; i < 16; i += 2)\n                qdata[n * (K / 2) + 8 * g + i / 2] = (uint8_t)(c[i + 1] | (c[i] << 4));"),
 ("deq_s_f32", C, "const float s = or_bf16_to_f32(or_f32_to_bf16_rne(s_channel[n]));", "const float s = s_channel[n];"),
 ("ste_f32acc", C, "row[k] += g * (double)or_bf16_to_f32(wr[k]);", "row[k] = (float)(row[k] + g * (double)or_bf16_to_f32(wr[k]));"),
 ("ste_via_f32", C, "dx[m * K + k] = or_f64_to_bf16_rne(row[k]);", "dx[m * K + k] = or_f32_to_bf16_rne((float)row[k]);"),
 ("py_interleave", "oracle/__init__.py", "return np.ascontiguousarray(np.swapaxes(halves, 0, 1)).reshape(a.shape)", "return np.ascontiguousarray(halves).reshape(a.shape)"),
 ("py_mp", "oracle/__init__.py", "return 1 << max(0, (int(m) - 1).bit_length())", "return max(1, int(m))"),
]

EQUIVALENT = {
    "aq_clamp": "|r / scale| <= qmax * (1 + 2^-23) < qmax + 1/2 for every finite row, so the clamp never binds",
    "stoch_lo_clamp": "with lo = last the threshold exceeds nothing that matters: the final clamp maps "
                      "lo + (x > thr) back to last, the value the page's clamp gives",
    "als_den_floor": "a zero denominator can only occur in the first ALS pass (an all-zero group on a zero "
                     "level); the NaN scale it gives sends every code to index 0 and the second pass "
                     "restores the floor 1e-8, so the outputs agree",
}


def run_one(mut, work):
    name, path, old, new = mut
    d = os.path.join(work, "m_" + name)
    if os.path.exists(d):
        shutil.rmtree(d)
    os.makedirs(d)
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(d, "oracle"),
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    shutil.copytree(os.path.join(ROOT, "tests"), os.path.join(d, "tests"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), d)
    os.symlink(os.path.join(ROOT, "w4a8_codebook_quantized_b200"), os.path.join(d, "w4a8_codebook_quantized_b200"))
    target = os.path.join(d, path)
    with open(target) as f:
        text = f.read()
    if text.count(old) != 1:
        return name, "NOT APPLIED", f"pattern found {text.count(old)} times"
    with open(target, "w") as f:
        f.write(text.replace(old, new))
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-q", "-x", "-m", "not gpu"],
                       cwd=d, capture_output=True, text=True, timeout=1200)
    failed = [ln for ln in r.stdout.splitlines() if ln.startswith(("FAILED", "ERROR"))]
    last = r.stdout.strip().splitlines()[-1] if r.stdout.strip() else r.stderr[-200:]
    return name, "CAUGHT" if r.returncode != 0 else "SURVIVED", failed[0] if failed else last


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--work", default=None, help="scratch directory for the mutated copies")
    ap.add_argument("--jobs", type=int, default=6)
    ap.add_argument("names", nargs="*")
    args = ap.parse_args()
    work = args.work or tempfile.mkdtemp(prefix="oracle_mutants_")
    os.makedirs(work, exist_ok=True)
    muts = [m for m in MUTATIONS if not args.names or m[0] in args.names]
    bad = 0
    with ThreadPoolExecutor(args.jobs) as ex:
        for name, status, info in ex.map(lambda m: run_one(m, work), muts):
            note = ""
            if status == "SURVIVED" and name in EQUIVALENT:
                status, note = "EQUIVALENT", EQUIVALENT[name]
            elif status != "CAUGHT":
                bad += 1
            print(f"{status:11s} {name:18s} {note or info[:110]}", flush=True)
    print(f"{len(muts)} mutations, {bad} neither caught nor equivalent")
    return 1 if bad else 0


if __name__ == "__main__":
    sys.exit(main())
