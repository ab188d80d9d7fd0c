/*
 * q8 oracle -- a plain, slow CPU statement of the 8-bit quantized linear layer.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark load this file.  It shares no code, header or table
 * with the CUDA library, and the CUDA library never calls it.
 *
 * Every step follows a formula the pages print; the citation sits on each
 * function.  Page short names used below:
 *   [Fabric]   "8-Bit LLM Quantization with Lightning Fabric" (mlqm.cn article)
 *   [CSDN]     "大模型量化技术" overview (devpress.csdn.net), sections 2.1-2.3
 *   [FBGEMM]   "Transformers FP8 (W8A8) 量化实战：基于 FBGEMM", sections 5.1-5.3, 6
 *   [LLM.int8] "Transformers 单 GPU 高效推理：bitsandbytes LLM.int8 8-bit 混合精度量化"
 *   [Xilyfe]   "大模型量化" blog (xilyfe.github.io), symmetric / asymmetric / INT32 /
 *              GGUF (block and Q4_K) sections
 *
 * Arithmetic rules (no fused multiply-add, no fast-math; build flags
 * -O2 -ffp-contract=off):
 *   - fp32 steps are written with C `float` operands, each one IEEE
 *     round-to-nearest-even, in the order the formula gives;
 *   - rne() rounds half to even, from its definition;
 *   - integer dot products accumulate in int64;
 *   - fp8 and fp16 dot products accumulate in double, then round once to fp32;
 *   - 16-bit and 8-bit float encodings are found by searching the format's
 *     sorted table of finite values (decoded from the format definition) for
 *     the nearest one, ties to the even code.
 *
 * Parity status: every exported function is pinned by tests/test_oracle_*.py
 * against closed forms, the pages' worked examples, brute force or an
 * independent library routine.  None is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_EPS 1e-8f /* QuantConfig eps, [Xilyfe] QuantInt8 sketch: scale.clamp(min=eps) */

/* ------------------------------------------------------------------------ */
/* Float formats, decoded from their definitions.                          */
/* ------------------------------------------------------------------------ */

enum { OR_F16 = 0, OR_BF16 = 1, OR_E4M3 = 2 };

/* IEEE 754 binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
static double dec_f16(uint32_t h) {
    uint32_t s = (h >> 15) & 1, e = (h >> 10) & 31, f = h & 1023;
    double v;
    if (e == 0) v = ldexp((double)f, -24);                  /* f/1024 * 2^-14 */
    else if (e == 31) v = f ? NAN : INFINITY;
    else v = ldexp((double)(1024 + f), (int)e - 25);         /* (1+f/1024) 2^(e-15) */
    return s ? -v : v;
}

/* bfloat16: the upper half of binary32; 8 exponent (bias 127), 7 fraction bits. */
static double dec_bf16(uint32_t b) {
    uint32_t s = (b >> 15) & 1, e = (b >> 7) & 255, f = b & 127;
    double v;
    if (e == 0) v = ldexp((double)f, -133);                 /* f/128 * 2^-126 */
    else if (e == 255) v = f ? NAN : INFINITY;
    else v = ldexp((double)(128 + f), (int)e - 134);         /* (1+f/128) 2^(e-127) */
    return s ? -v : v;
}

/* OCP FP8 E4M3 ("fn"): 4 exponent (bias 7), 3 fraction bits, no infinities;
 * exponent 15 with fraction 7 is NaN, so the largest finite value is 448
 * ([FBGEMM] 4-bit exponent + 3-bit mantissa float8_e4m3fn storage). */
static double dec_e4m3(uint32_t c) {
    uint32_t s = (c >> 7) & 1, e = (c >> 3) & 15, f = c & 7;
    double v;
    if (e == 15 && f == 7) v = NAN;
    else if (e == 0) v = ldexp((double)f, -9);               /* f/8 * 2^-6 */
    else v = ldexp((double)(8 + f), (int)e - 10);            /* (1+f/8) 2^(e-7) */
    return s ? -v : v;
}

/* Sorted non-negative finite values of each format, indexed by code. */
static double *g_tab[3];
static uint32_t g_tab_n[3];
static double g_e4m3_signed[256]; /* every E4M3 code, sign included (NaN codes too) */

static void build_tables(void) {
    if (g_tab[0]) return;
    uint32_t nf16 = 0x7BFF + 1, nbf = 0x7F7F + 1, ne4 = 0x7E + 1;
    double *t0 = malloc(sizeof(double) * nf16), *t1 = malloc(sizeof(double) * nbf),
           *t2 = malloc(sizeof(double) * ne4);
    for (uint32_t c = 0; c < nf16; ++c) t0[c] = dec_f16(c);
    for (uint32_t c = 0; c < nbf; ++c) t1[c] = dec_bf16(c);
    for (uint32_t c = 0; c < ne4; ++c) t2[c] = dec_e4m3(c);
    for (uint32_t c = 0; c < 256; ++c) g_e4m3_signed[c] = dec_e4m3(c);
    g_tab_n[0] = nf16; g_tab_n[1] = nbf; g_tab_n[2] = ne4;
    g_tab[1] = t1; g_tab[2] = t2;
    g_tab[0] = t0; /* last: marks the tables ready */
}

/* Nearest code to |v| in format `fmt`, ties to the even code.  Beyond the
 * largest finite value, IEEE formats round to infinity at or past the
 * midpoint to 2^(emax+1); E4M3 saturates to 448 (satfinite). */
static uint32_t enc_format(double v, int fmt) {
    const double *t = g_tab[fmt];
    uint32_t n = g_tab_n[fmt];
    uint32_t sign = signbit(v) ? 1u : 0u;
    uint32_t sbit = fmt == OR_E4M3 ? 0x80u : 0x8000u;
    if (isnan(v)) return fmt == OR_F16 ? 0x7E00u : fmt == OR_BF16 ? 0x7FC0u : 0x7Fu;
    double a = fabs(v);
    uint32_t code;
    if (a >= t[n - 1]) {
        if (fmt == OR_E4M3) code = n - 1;
        else {
            double next = fmt == OR_F16 ? 65536.0 : ldexp(1.0, 128);
            double mid = 0.5 * (t[n - 1] + next);
            code = a >= mid ? n : n - 1;  /* code n is +inf: 0x7C00 / 0x7F80 */
        }
    } else {
        uint32_t lo = 0, hi = n - 1;      /* t[lo] <= a < t[hi] */
        while (hi - lo > 1) {
            uint32_t mid = lo + (hi - lo) / 2;
            if (t[mid] <= a) lo = mid; else hi = mid;
        }
        double dlo = a - t[lo], dhi = t[hi] - a;
        if (dlo < dhi) code = lo;
        else if (dhi < dlo) code = hi;
        else code = (lo % 2 == 0) ? lo : hi;
    }
    return code | (sign ? sbit : 0u);
}

void or_init(void) { build_tables(); }

int or_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void or_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* 16-bit patterns (fmt F16 or BF16) -> exact fp32 values. */
void or_widen16(const uint16_t *in, int fmt, float *out, int64_t n) {
    for (int64_t i = 0; i < n; ++i)
        out[i] = (float)(fmt == OR_F16 ? dec_f16(in[i]) : dec_bf16(in[i]));
}

/* E4M3 codes -> exact fp32 values. */
void or_widen_e4m3(const uint8_t *in, float *out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = (float)dec_e4m3(in[i]);
}

/* fp32 -> 16-bit pattern (F16 or BF16), round to nearest even. */
void or_round16(const float *in, int fmt, uint16_t *out, int64_t n) {
    build_tables();
    for (int64_t i = 0; i < n; ++i) out[i] = (uint16_t)enc_format((double)in[i], fmt);
}

/* fp32 -> E4M3 code, round to nearest even, saturating at +-448. */
void or_round_e4m3(const float *in, uint8_t *out, int64_t n) {
    build_tables();
    for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)enc_format((double)in[i], OR_E4M3);
}

/* Round half to even, from the definition (|v| < 2^52). */
static double rne(double v) {
    double f = floor(v), d = v - f;
    if (d > 0.5) return f + 1.0;
    if (d < 0.5) return f;
    return fmod(f, 2.0) == 0.0 ? f : f + 1.0;
}

static double clampd(double v, double lo, double hi) { return v < lo ? lo : v > hi ? hi : v; }

/* ------------------------------------------------------------------------ */
/* Weight quantization, one row (output channel) at a time.                 */
/* ------------------------------------------------------------------------ */

/*
 * Per-output-channel asymmetric quantization with b-bit signed codes.
 * [Xilyfe] asymmetric section: s = (2^b - 1)/(alpha - beta) as a multiplier,
 * z = round(-s*beta) - 2^(b-1), x_int = round(s*x + z); stored here as the
 * dequant multiplier S = (alpha - beta)/(2^b - 1) so that r = S (q - Z)
 * ([Xilyfe] "量化是什么": r = S x (q - Z); [CSDN] 2.1: Q = round(R/S) + Z;
 * [CSDN] 2.3 min-max: S = (Rmax - Rmin)/(Qmax - Qmin), Z = Qmin - round(Rmin/S);
 * [Fabric] 2.1 / 2.3: one scale and zero point per row, scale = (b - a)/255).
 * Per row: beta = min, alpha = max;
 *   S = fl32(fl32(alpha - beta) / (2^b - 1)), clamped below at eps;
 *   Z = clamp(rne(fl32(-beta / S)) - 2^(b-1), qmin, qmax);
 *   q = clamp(rne(fl32(w / S)) + Z, qmin, qmax).
 * q, S, Z are written per row; Z is an integer held in fp32.
 */
void or_quant_weight_asym(const float *W, int64_t n, int64_t k, int bits,
                          int8_t *q, float *S, float *Z) {
    const double qmin = -ldexp(1.0, bits - 1), qmax = ldexp(1.0, bits - 1) - 1.0;
    const float levels = (float)(ldexp(1.0, bits) - 1.0);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        const float *w = W + r * k;
        float lo = w[0], hi = w[0];
        for (int64_t j = 1; j < k; ++j) {
            if (w[j] < lo) lo = w[j];
            if (w[j] > hi) hi = w[j];
        }
        float range = hi - lo;
        float s = range / levels;
        if (!(s >= OR_EPS)) s = OR_EPS;
        float zq = -lo / s;
        double z = clampd(rne((double)zq) + qmin, qmin, qmax);
        for (int64_t j = 0; j < k; ++j) {
            float t = w[j] / s;
            q[r * k + j] = (int8_t)clampd(rne((double)t) + z, qmin, qmax);
        }
        S[r] = s;
        Z[r] = (float)z;
    }
}

/*
 * Per-output-channel symmetric quantization with b-bit codes in [-qmax, qmax],
 * qmax = 2^(b-1) - 1.  [Xilyfe] symmetric section: alpha = max |x|,
 * s = (2^(b-1) - 1)/alpha, x_int = round(s x); stored as S = alpha/qmax with
 * q = rne(fl32(w / S)); the clamp to +-qmax and the eps floor follow the
 * [Xilyfe] QuantInt8._quantize sketch.  Worked examples with b = 4 sit in the
 * [Xilyfe] GGUF section.
 */
/* One block of `len` weights: S = fl32(max|w| / qmax), eps floor,
 * q = clamp(rne(fl32(w / S)), -qmax, qmax). */
static void sym_block(const float *w, int64_t len, double qmax, int8_t *q, float *S) {
    float a = 0.0f;
    for (int64_t j = 0; j < len; ++j) {
        float v = fabsf(w[j]);
        if (v > a) a = v;
    }
    float s = a / (float)qmax;
    if (!(s >= OR_EPS)) s = OR_EPS;
    for (int64_t j = 0; j < len; ++j) {
        float t = w[j] / s;
        q[j] = (int8_t)clampd(rne((double)t), -qmax, qmax);
    }
    *S = s;
}

void or_quant_weight_sym(const float *W, int64_t n, int64_t k, int bits,
                         int8_t *q, float *S) {
    const double qmax = ldexp(1.0, bits - 1) - 1.0;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) sym_block(W + r * k, k, qmax, q + r * k, &S[r]);
}

/*
 * Group-wise symmetric b-bit weights.  [CSDN] 2.2 (granularity table): one
 * scale per group of 64-128 consecutive parameters; [Xilyfe] GGUF section:
 * the row is cut into blocks and each block gets its own absmax scale, with
 * qmax = 2^(b-1) - 1 (7 for 4 bits).  Every group of g consecutive weights
 * along a row is one block of the symmetric rule above.  S is n x (k / g),
 * row-major: S[r * (k / g) + j] belongs to weights r, j*g .. j*g + g - 1.
 */
void or_quant_weight_group(const float *W, int64_t n, int64_t k, int bits, int64_t g,
                           int8_t *q, float *S) {
    const double qmax = ldexp(1.0, bits - 1) - 1.0;
    const int64_t ng = k / g;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r)
        for (int64_t j = 0; j < ng; ++j)
            sym_block(W + r * k + j * g, g, qmax, q + r * k + j * g, &S[r * ng + j]);
}

/*
 * GGUF Q4_K-style two-level scales ([Xilyfe] GGUF section, Q4_K simulation):
 * a super block is 8 sub-blocks of 32 weights along a row.  Each sub-block is
 * one symmetric 4-bit block (or_quant_weight_group with g = 32: s_sub =
 * absmax / 7, codes from the unquantized s_sub, as the page's step 3 does);
 * then the 8 sub-block scales are quantized like a second set of weights by
 * absmax over 15 levels (they are never negative):
 *   s_super = fl32(max_j s_sub[j] / 15),
 *   q_sub[j] = clamp(rne(fl32(s_sub[j] / s_super)), 0, 15),
 * and the scale a sub-block is dequantized with is
 *   S_eff[j] = fl32(s_super * q_sub[j]).
 * Layouts: q n x k; s_sub, q_sub, S_eff n x (k / 32); s_super n x (k / 256).
 */
void or_quant_weight_q4k(const float *W, int64_t n, int64_t k, int8_t *q, float *s_sub,
                         float *s_super, uint8_t *q_sub, float *S_eff) {
    const int64_t ns = k / 32, nb = k / 256;
    or_quant_weight_group(W, n, k, 4, 32, q, s_sub);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r)
        for (int64_t b = 0; b < nb; ++b) {
            const float *ss = s_sub + r * ns + b * 8;
            float mx = ss[0];
            for (int j = 1; j < 8; ++j)
                if (ss[j] > mx) mx = ss[j];
            float sup = mx / 15.0f;
            s_super[r * nb + b] = sup;
            for (int j = 0; j < 8; ++j) {
                float t = ss[j] / sup;
                double c = clampd(rne((double)t), 0.0, 15.0);
                q_sub[r * ns + b * 8 + j] = (uint8_t)c;
                S_eff[r * ns + b * 8 + j] = sup * (float)c;
            }
        }
}

/*
 * The 16-bit weight a group-quantized layer multiplies when its activations
 * are 16-bit (W4A16: the weight is brought back to the activation's format,
 * r = S q, [Xilyfe] "量化是什么" with Z = 0):
 * out[r, j] = round16(fl32(S[r, j / g] * q[r, j]), fmt), fmt 0 fp16, 1 bf16.
 */
void or_dequant_group16(const int8_t *q, const float *S, int64_t n, int64_t k, int64_t g,
                        int fmt, uint16_t *out) {
    build_tables();
    const int64_t ng = k / g;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r)
        for (int64_t j = 0; j < k; ++j) {
            float v = S[r * ng + j / g] * (float)q[r * k + j];
            out[r * k + j] = (uint16_t)enc_format((double)v, fmt == 0 ? OR_F16 : OR_BF16);
        }
}

/*
 * Per-output-channel FP8 E4M3 weights with one fp32 scale per row
 * ([FBGEMM] 5.1: weight float8_e4m3fn (out, in), weight_scale fp32 (out, 1)).
 * S = fl32(max|w| / 448) with the eps floor; q = e4m3_rne_satfinite(fl32(w / S)).
 */
void or_quant_weight_fp8(const float *W, int64_t n, int64_t k, uint8_t *q, float *S) {
    build_tables();
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        const float *w = W + r * k;
        float a = 0.0f;
        for (int64_t j = 0; j < k; ++j) {
            float v = fabsf(w[j]);
            if (v > a) a = v;
        }
        float s = a / 448.0f;
        if (!(s >= OR_EPS)) s = OR_EPS;
        for (int64_t j = 0; j < k; ++j) {
            float t = w[j] / s;
            q[r * k + j] = (uint8_t)enc_format((double)t, OR_E4M3);
        }
        S[r] = s;
    }
}

/* ------------------------------------------------------------------------ */
/* Activation quantization, one row (token) at a time, every call.          */
/* ------------------------------------------------------------------------ */

/*
 * Dynamic per-token symmetric INT8 ([Xilyfe] symmetric section and dynamic
 * quantization paragraph; [FBGEMM] 5.2 per-row activation scale).
 * Columns with skip[k] != 0 (the LLM.int8 outlier set) are left out: alpha is
 * the max over the other columns and their codes are 0 ([LLM.int8] 核心思想:
 * the regular stream is "the rest").
 *   S = max(fl32(alpha / 127), eps); q = clamp(rne(fl32(x / S)), -127, 127);
 *   rowsum = sum_k q (int32), used by the zero-point correction.
 */
void or_quant_act_int8(const float *X, int64_t m, int64_t k, const uint8_t *skip,
                       int8_t *q, float *S, int32_t *rowsum) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < m; ++r) {
        const float *x = X + r * k;
        float a = 0.0f;
        for (int64_t j = 0; j < k; ++j) {
            if (skip && skip[j]) continue;
            float v = fabsf(x[j]);
            if (v > a) a = v;
        }
        float s = a / 127.0f;
        if (!(s >= OR_EPS)) s = OR_EPS;
        int64_t sum = 0;
        for (int64_t j = 0; j < k; ++j) {
            int8_t c = 0;
            if (!(skip && skip[j])) {
                float t = x[j] / s;
                c = (int8_t)clampd(rne((double)t), -127.0, 127.0);
            }
            q[r * k + j] = c;
            sum += c;
        }
        S[r] = s;
        if (rowsum) rowsum[r] = (int32_t)sum;
    }
}

/*
 * Dynamic per-token INT8 quantization of a smoothed activation ("大模型量化"
 * (Xilyfe), algorithm list, SmoothQuant: the activation's outlier channels are
 * "smoothed" onto the weight side so the activation quantizes easily; the page
 * gives no formula).  Reading: per input column j a smoothing factor s_j is
 * chosen offline; the activation is divided by it and the weight column
 * multiplied by it, which leaves X W^T unchanged.  The division is applied as
 * a multiplier m_j = RN(1/s_j) supplied by the caller: xs = fl32(x * m_j), then
 * the dynamic symmetric INT8 quantizer of or_quant_act_int8 runs on xs.  The
 * weight side, fl32(w * s_j), is plain offline preprocessing (or_smooth_weight).
 */
void or_quant_act_smooth(const float *X, int64_t m, int64_t k, const float *mult, int8_t *q,
                         float *S, int32_t *rowsum) {
    float *xs = (float *)malloc((size_t)(m * k) * sizeof(float));
    for (int64_t r = 0; r < m; ++r)
        for (int64_t j = 0; j < k; ++j) xs[r * k + j] = X[r * k + j] * mult[j];
    or_quant_act_int8(xs, m, k, NULL, q, S, rowsum);
    free(xs);
}

void or_smooth_weight(const float *W, int64_t n, int64_t k, const float *s, float *out) {
    for (int64_t r = 0; r < n; ++r)
        for (int64_t j = 0; j < k; ++j) out[r * k + j] = W[r * k + j] * s[j];
}

/*
 * Static (calibrated) symmetric INT8 quantization with one scale for the
 * whole tensor ("大模型量化" (Xilyfe), the paragraph on 静态量化: the scale is
 * worked out once from a calibration pass and reused on every call instead of
 * being recomputed from each input).  Reading: symmetric, per-tensor, the
 * caller passes S > 0; q = clamp(rne(fl32(x / S)), -127, 127), so inputs
 * beyond 127 S saturate, as the code range of every other quantizer here.
 * S is copied to every row's scale so the result feeds the W8A8 linear like
 * a dynamic activation; rowsum[r] = sum of the row's codes (for asymmetric
 * weights).
 */
static int8_t static_code(float x, float S) {
    const float t = x / S;
    return (int8_t)clampd(rne((double)t), -127.0, 127.0);
}

void or_quant_act_static(const float *X, int64_t m, int64_t k, float S, int8_t *q, float *Sout,
                         int32_t *rowsum) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < m; ++r) {
        int64_t sum = 0;
        for (int64_t j = 0; j < k; ++j) {
            const int8_t c = static_code(X[r * k + j], S);
            q[r * k + j] = c;
            sum += c;
        }
        Sout[r] = S;
        if (rowsum) rowsum[r] = (int32_t)sum;
    }
}

/*
 * Re-quantization of a layer's output for the next layer ("大模型量化"
 * (Xilyfe), 量化对象 section, INT8 这么小的范围不会导致溢出吗: after the INT32
 * accumulation the result is scaled back into INT8 before it is passed on).
 * Reading: the fp32 output y of the dequant epilogue (bias included) is
 * quantized with the next layer's static input scale S_out:
 * q = clamp(rne(fl32(y / S_out)), -127, 127).
 */
void or_requant(const float *y, int64_t count, float S, int8_t *q) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) q[i] = static_code(y[i], S);
}

/*
 * Dynamic per-token FP8 E4M3 with an upper bound on the row scale
 * ([FBGEMM] 5.2 and 6: quantize_fp8_per_row clips the input at
 * activation_scale_ub, default 1200.0).  alpha = min(max|x|, ub) when ub > 0;
 * S = max(fl32(alpha / 448), eps); q = e4m3_rne_satfinite(fl32(x / S)), so
 * entries beyond alpha saturate at +-448.
 */
void or_quant_act_fp8(const float *X, int64_t m, int64_t k, float ub, uint8_t *q, float *S) {
    build_tables();
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < m; ++r) {
        const float *x = X + r * k;
        float a = 0.0f;
        for (int64_t j = 0; j < k; ++j) {
            float v = fabsf(x[j]);
            if (v > a) a = v;
        }
        if (ub > 0.0f && a > ub) a = ub;
        float s = a / 448.0f;
        if (!(s >= OR_EPS)) s = OR_EPS;
        for (int64_t j = 0; j < k; ++j) {
            float t = x[j] / s;
            q[r * k + j] = (uint8_t)enc_format((double)t, OR_E4M3);
        }
        S[r] = s;
    }
}

/*
 * LLM.int8 outlier feature columns ([LLM.int8] 核心思想 and BitsAndBytesConfig
 * table: llm_int8_threshold = 6.0, values beyond it take the fp16 stream).
 * Column k is an outlier when some token has |x| strictly above T.  T <= 0
 * turns the decomposition off (no outliers).  Writes mask[k] in {0, 1}, the
 * outlier columns in ascending order into idx[0 .. count), and count.
 */
void or_outlier_columns(const float *X, int64_t m, int64_t k, float T,
                        uint8_t *mask, int32_t *idx, int32_t *count) {
    int32_t c = 0;
    for (int64_t j = 0; j < k; ++j) {
        int out = 0;
        if (T > 0.0f)
            for (int64_t r = 0; r < m && !out; ++r)
                if (fabsf(X[r * k + j]) > T) out = 1;
        mask[j] = (uint8_t)out;
        if (out) idx[c++] = (int32_t)j;
    }
    *count = c;
}

/* ------------------------------------------------------------------------ */
/* GEMMs and epilogues, over a chosen set of output rows and columns.       */
/* ------------------------------------------------------------------------ */

/*
 * INT8 x INT8 dot products with a wide accumulator ([Xilyfe] "INT8 这么小的范围
 * 不会导致溢出吗": products accumulate in INT32).  Accumulates in int64 so the
 * caller can check that the INT32 bound holds.  A is M x K (token codes), B is
 * N x K (weight codes), both row-major; *_signed selects int8 or uint8 codes.
 * acc[i * nc + j] = sum_k A[rows[i], k] * B[cols[j], k].
 */
void or_gemm_int(const void *A, int a_signed, int64_t lda, const void *B, int b_signed,
                 int64_t ldb, int64_t k, const int64_t *rows, int64_t nr,
                 const int64_t *cols, int64_t nc, int64_t *acc) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nr; ++i) {
        const int8_t *as = (const int8_t *)A + rows[i] * lda;
        const uint8_t *au = (const uint8_t *)A + rows[i] * lda;
        for (int64_t j = 0; j < nc; ++j) {
            const int8_t *bs = (const int8_t *)B + cols[j] * ldb;
            const uint8_t *bu = (const uint8_t *)B + cols[j] * ldb;
            int64_t s = 0;
            for (int64_t t = 0; t < k; ++t) {
                int64_t a = a_signed ? (int64_t)as[t] : (int64_t)au[t];
                int64_t b = b_signed ? (int64_t)bs[t] : (int64_t)bu[t];
                s += a * b;
            }
            acc[i * nc + j] = s;
        }
    }
}

/*
 * Dequant epilogue of the quantized matmul.  With R = S (Q - Z)
 * ([Xilyfe] "量化是什么"; [CSDN] 2.1 quantized matmul, its "Z + Q" sign read
 * as "Q - Z"), and activations symmetric (Z_x = 0):
 *   y = S_x S_w sum_k qx (qw - Zw) = S_x S_w (acc - Zw * rowsum).
 * fp32 order: c = acc - Zw[n] * rowsum[m] (exact integer), y = fl32(c),
 * y = fl32(y * S_x[m]), y = fl32(y * S_w[n]), then y = fl32(y + bias[n]) when a
 * bias is given ([FBGEMM] 5.3 and [LLM.int8]: the bias keeps its precision and
 * is added after the scaled product).  Zw may be NULL (symmetric weights).
 */
void or_epilogue_int(const int64_t *acc, const int64_t *rows, int64_t nr,
                     const int64_t *cols, int64_t nc, const float *Zw,
                     const int32_t *rowsum, const float *Sx, const float *Sw,
                     const float *bias, float *y) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nr; ++i)
        for (int64_t j = 0; j < nc; ++j) {
            int64_t m = rows[i], n = cols[j];
            int64_t c = acc[i * nc + j];
            if (Zw) c -= (int64_t)Zw[n] * (int64_t)rowsum[m];
            float v = (float)c;
            v = v * Sx[m];
            v = v * Sw[n];
            if (bias) v = v + bias[n];
            y[i * nc + j] = v;
        }
}

/*
 * FP8 rowwise GEMM ([FBGEMM] 5.3: f8f8bf16_rowwise(xq, w, x_scale, w_scale)
 * then + bias).  Products of the decoded E4M3 values are summed in double and
 * rounded once to fp32: acc; then y = fl32(fl32(acc * S_x[m]) * S_w[n]),
 * y = fl32(y + bias[n]) when a bias is given.
 */
void or_gemm_fp8(const uint8_t *A, int64_t lda, const uint8_t *B, int64_t ldb, int64_t k,
                 const int64_t *rows, int64_t nr, const int64_t *cols, int64_t nc,
                 const float *Sx, const float *Sw, const float *bias,
                 float *acc_out, float *y) {
    build_tables();
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nr; ++i) {
        const uint8_t *a = A + rows[i] * lda;
        for (int64_t j = 0; j < nc; ++j) {
            const uint8_t *b = B + cols[j] * ldb;
            double s = 0.0;
            for (int64_t t = 0; t < k; ++t) s += g_e4m3_signed[a[t]] * g_e4m3_signed[b[t]];
            float acc = (float)s;
            float v = acc * Sx[rows[i]];
            v = v * Sw[cols[j]];
            if (bias) v = v + bias[cols[j]];
            if (acc_out) acc_out[i * nc + j] = acc;
            y[i * nc + j] = v;
        }
    }
}

/*
 * The 16-bit weight the outlier stream multiplies, when only the 8-bit
 * weight is kept ([LLM.int8] BitsAndBytesConfig: llm_int8_has_fp16_weight
 * defaults to False; only `weight` is stored in 1 byte per parameter):
 * W16[n, k] = fp16_rne(fl32(S[n] * fl32(q[n, k] - Z[n]))), the dequant
 * r = S (q - Z) of [Xilyfe] "量化是什么" / [Fabric] 3.3 dequantize_weight.
 * Written only for the listed columns: W16 is nr x ncols, row-major.
 * q_signed selects int8 or uint8 codes; Z may be NULL (symmetric).
 */
void or_dequant_weight_f16(const void *q, int q_signed, int64_t ldq, const float *S,
                           const float *Z, const int64_t *rows, int64_t nr,
                           const int32_t *colidx, int64_t ncols, uint16_t *W16) {
    build_tables();
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nr; ++i) {
        int64_t n = rows[i];
        for (int64_t j = 0; j < ncols; ++j) {
            int64_t kk = colidx[j];
            float code = q_signed ? (float)((const int8_t *)q)[n * ldq + kk]
                                  : (float)((const uint8_t *)q)[n * ldq + kk];
            float d = Z ? code - Z[n] : code;
            float v = S[n] * d;
            W16[i * ncols + j] = (uint16_t)enc_format((double)v, OR_F16);
        }
    }
}

/*
 * Dequantized weight in fp32, r = fl32(S[n] * fl32(q - Z[n])) for every element
 * ([Xilyfe] "量化是什么": r = S (q - Z); [Fabric] 3.3 dequantize_weight).
 * code_kind: 0 int8, 1 uint8, 2 E4M3 (decoded exactly); Z may be NULL.
 */
void or_dequant_weight(const void *q, int code_kind, int64_t n, int64_t k, int64_t ldq,
                       const float *S, const float *Z, float *out) {
    build_tables();
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r)
        for (int64_t j = 0; j < k; ++j) {
            float code;
            if (code_kind == 0) code = (float)((const int8_t *)q)[r * ldq + j];
            else if (code_kind == 1) code = (float)((const uint8_t *)q)[r * ldq + j];
            else code = (float)g_e4m3_signed[((const uint8_t *)q)[r * ldq + j]];
            float d = Z ? code - Z[r] : code;
            out[r * k + j] = S[r] * d;
        }
}

/*
 * LLM.int8 outlier stream ([LLM.int8] 核心思想: columns beyond the threshold
 * are multiplied in fp16): y16[m, n] = fl32(sum_{j < count} X[m, idx[j]] *
 * W16[n, j]), products and sum in double.  X is the full M x K activation
 * (fp32 holding fp16 values); W16 is the row-major N x count fp16-valued
 * matrix of the outlier columns (fp32 holding fp16 values), rows indexed by
 * cols[] through its leading dimension ldw.
 */
void or_outlier_gemm(const float *X, int64_t ldx, const float *W16, int64_t ldw,
                     const int32_t *idx, int64_t count, const int64_t *rows, int64_t nr,
                     const int64_t *cols, int64_t nc, float *y16) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nr; ++i)
        for (int64_t j = 0; j < nc; ++j) {
            double s = 0.0;
            for (int64_t t = 0; t < count; ++t)
                s += (double)X[rows[i] * ldx + idx[t]] * (double)W16[cols[j] * ldw + t];
            y16[i * nc + j] = (float)s;
        }
}

/* y = fl32(a + b) elementwise: the merge of the two LLM.int8 streams, then an
 * optional bias per column (cols[] indexes bias): y = fl32(y + bias[n]). */
void or_merge(const float *a, const float *b, int64_t nr, const int64_t *cols, int64_t nc,
              const float *bias, float *y) {
    for (int64_t i = 0; i < nr; ++i)
        for (int64_t j = 0; j < nc; ++j) {
            float v = a[i * nc + j] + b[i * nc + j];
            if (bias) v = v + bias[cols[j]];
            y[i * nc + j] = v;
        }
}
