/*
 * moe_oracle.c -- the CPU oracle for the routed-MoE SwiGLU expert forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no source, header, table or
 * helper with the CUDA library; it is written from the pages' description
 * of what the method computes, one token at a time, in double precision
 * wherever the pages do not fix a narrower type.
 *
 * What each function follows (page title, section):
 *   oracle_route       -- "core.transformer.moe.training_matches_inference"
 *                         API doc, `_route` (top-k probs and ids per token),
 *                         and Megatron-LM PR #7830 "Mega backend for
 *                         generation" (expert ids put in a canonical sorted
 *                         order before the combine).  Softmax over the
 *                         experts, top-k, the k probabilities renormalised to
 *                         sum to one; ties go to the lower expert id.
 *   oracle_permute     -- same API doc, `expert_value_pass` ("each row is one
 *                         route, sorted by local expert"); rows stable by
 *                         token inside an expert.
 *   oracle_mxfp8_*     -- Megatron-LM PR #7830 (mxfp8_quantize_per_block_32)
 *                         and cudnn-frontend PR #448 review of the MXFP8
 *                         block contract (32-element blocks): E4M3 elements,
 *                         one E8M0 power-of-two scale per 32 elements along
 *                         K, the OCP MX rule scale = 2^(floor(log2 amax)-8),
 *                         round-to-nearest-even, saturating to +-448.
 *   oracle_nvfp4_*     -- Megatron-LM PR #7798, "Per-token NVFP4" and
 *                         "Core metric" (TE's per-token recipe:
 *                         NVFP4BlockScaling with row-scaled activations, 1-D
 *                         blocks, no Hadamard transform, no stochastic
 *                         rounding): E2M1 elements, one E4M3 scale per 16
 *                         elements along K, and an fp32 second-level scale
 *                         per activation row (per weight matrix for weights).
 *                         The pages give the recipe's name, not its formulas;
 *                         the reading taken is written out at nvfp4_row().
 *   oracle_forward_*   -- Megatron-LM PR #7798, "Background" (activation
 *                         fused into FC1, probabilities applied after FC2)
 *                         and "What is changed" (a token's routes summed as
 *                         fp32 fused multiply-adds of probability and row,
 *                         starting from zero, in the listed order); PR #8367
 *                         "Problem" (the result is returned in fp32, no bf16
 *                         downcast).  SwiGLU: h = silu(gate . x) * (up . x).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - probabilities are renormalised over the k chosen experts in every
 *     configuration;
 *   - the combine order is ascending expert id;
 *   - the expert output row y stays fp32 (the FC2 accumulator) before the
 *     combine, and the combine output is not rounded to bf16;
 *   - the SwiGLU intermediate is computed in double, rounded to fp32, then to
 *     bf16 (round-to-nearest-even) or re-quantised to MXFP8 exactly as the
 *     kernel path does;
 *   - an all-zero MXFP8 block gets scale byte 0 (2^-127); negative values
 *     that round to zero keep their sign (code 0x80).
 *
 * Variants (cudnn-frontend PR #448, the MoeEp constructor's options;
 * Megatron-LM PR #8367 for the finalize's output type), each off by default:
 *   ORACLE_PROBS_IN_FC1 -- `apply_topk_in_fc1`: the route's probability
 *       multiplies the SwiGLU row before it is rounded for FC2,
 *       h_f = round(fp32(p_j * silu(g_f) * u_f)), and the combine adds the
 *       routes' rows as fp32 additions from 0.0f in ascending id.
 *   clamp > 0          -- `gate_up_clamp`: the gate and up pre-activations
 *       (the FC1 accumulator) are clamped to [-clamp, clamp] before SwiGLU.
 *   oracle_round_bf16  -- a bf16 finalize output: the fp32 sum rounded to
 *       bf16 (round-to-nearest-even), as the pages' BF16 finalize does.
 *   ORACLE_SQUARED_RELU -- squared-ReLU experts (the Nano-v3 shapes of
 *       Megatron-LM PR #8367's measurements and the nvfp4-squared_relu
 *       recipe of its tests): one FC1 projection W1 = w_gate [E, F, H], no
 *       up projection, h_f = round(fp32(relu(g_f)^2)); the clamp and the
 *       probability in FC1 act on g_f and on the row as above.
 *   The pages name these options but give no formula; the readings above
 *   are the plainest ones and are listed in the design notes.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC (no -ffast-math: fmaf and the
 * double sums must keep IEEE semantics).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_ENOMEM 2

/* ------------------------------------------------------------------ */
/* Number formats                                                      */
/* ------------------------------------------------------------------ */

/* bf16 bit pattern -> float (exact: bf16 is the top half of an fp32). */
static float bf16_bits_to_float(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* float -> bf16 with round-to-nearest-even on the 16 dropped bits.  The
 * inputs here are finite; a NaN stays a quiet NaN. */
static uint16_t float_to_bf16_bits_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) {
        return (uint16_t)((u >> 16) | 0x0040u);
    }
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* E4M3 (OCP FP8, "fn" flavour: no infinities, S.1111.111 is NaN).
 * Value of a code from the format definition: bias 7, subnormals when the
 * exponent field is zero with step 2^-9. */
static double e4m3_code_value(int code) {
    int sign = (code >> 7) & 1;
    int ef = (code >> 3) & 15;
    int mf = code & 7;
    double mag;
    if (ef == 15 && mf == 7) return NAN;
    if (ef == 0)
        mag = ldexp((double)mf, -9);
    else
        mag = ldexp(1.0 + mf / 8.0, ef - 7);
    return sign ? -mag : mag;
}

/* The 127 finite non-negative codes 0x00..0x7e have strictly increasing
 * values, so the nearest grid point of a magnitude is found by bisection
 * over this table. */
static double g_e4m3_mag[127];
static double g_e4m3_all[256];
static double g_pow2[256]; /* g_pow2[b] = 2^(b-127), the E8M0 scale value */
static int g_tables_ready = 0;

static void build_tables(void) {
    if (g_tables_ready) return;
    for (int c = 0; c < 127; ++c) g_e4m3_mag[c] = e4m3_code_value(c);
    for (int c = 0; c < 256; ++c) g_e4m3_all[c] = e4m3_code_value(c);
    for (int b = 0; b < 256; ++b) g_pow2[b] = ldexp(1.0, b - 127);
    g_tables_ready = 1;
}

/* Round a real value onto the E4M3 grid: nearest code, ties to the code
 * with an even mantissa LSB, magnitudes beyond 448 saturate to 448, the
 * sign is kept (so -tiny -> 0x80). */
static uint8_t e4m3_encode_rne_sat(double v) {
    int neg = signbit(v) ? 1 : 0;
    double a = fabs(v);
    int code;
    if (a >= g_e4m3_mag[126]) {
        code = 126; /* 448: saturate */
    } else {
        /* largest lo with mag[lo] <= a */
        int lo = 0, hi = 126;
        while (hi - lo > 1) {
            int mid = (lo + hi) / 2;
            if (g_e4m3_mag[mid] <= a) lo = mid; else hi = mid;
        }
        double dlo = a - g_e4m3_mag[lo];
        double dhi = g_e4m3_mag[hi] - a;
        if (dlo < dhi) code = lo;
        else if (dhi < dlo) code = hi;
        else code = (lo & 1) ? hi : lo; /* tie: even mantissa */
    }
    return (uint8_t)(code | (neg << 7));
}

/* OCP MX shared-scale exponent of one block from its largest magnitude:
 * floor(log2(amax)) - emax(E4M3)=8, clamped to the E8M0 range; an all-zero
 * block gets the smallest scale.  Returns the biased byte. */
static uint8_t e8m0_block_scale(double amax) {
    int s;
    if (amax == 0.0) {
        s = -127;
    } else {
        int ex;
        (void)frexp(amax, &ex);      /* amax = m * 2^ex, m in [0.5, 1) */
        s = (ex - 1) - 8;            /* floor(log2 amax) - 8 */
        if (s < -127) s = -127;
        if (s > 127) s = 127;
    }
    return (uint8_t)(s + 127);
}

/* Quantise n values (n <= 32, one block) into codes + one scale byte. */
static void mxfp8_block(const double* v, int n, uint8_t* q, uint8_t* sbyte) {
    double amax = 0.0;
    for (int i = 0; i < n; ++i) {
        double a = fabs(v[i]);
        if (a > amax) amax = a;
    }
    uint8_t sb = e8m0_block_scale(amax);
    double inv = ldexp(1.0, -((int)sb - 127)); /* exact power of two */
    for (int i = 0; i < n; ++i) q[i] = e4m3_encode_rne_sat(v[i] * inv);
    *sbyte = sb;
}

/* E2M1 (FP4: 1 sign, 2 exponent, 1 mantissa bit, bias 1): code c = 0..7
 * of a magnitude from the format definition: subnormal 0.5 * m when the
 * exponent field is 0, else (1 + m / 2) * 2^(e - 1); no infinities, no NaN. */
static double e2m1_code_value(int code) {
    int ef = (code >> 1) & 3, mf = code & 1;
    double mag = ef == 0 ? 0.5 * mf : ldexp(1.0 + 0.5 * mf, ef - 1);
    return (code & 8) ? -mag : mag;
}

/* Round a real value onto the E2M1 grid: nearest magnitude, ties to the
 * code with an even mantissa bit, magnitudes beyond 6 (and NaN) saturate to
 * 6, the sign is kept (so -tiny -> code 8). */
static uint8_t e2m1_encode_rne_sat(double v) {
    int neg = signbit(v) ? 1 : 0;
    double a = fabs(v);
    int code;
    if (!(a < 6.0)) {
        code = 7;
    } else {
        int lo = 0, hi = 7;
        while (hi - lo > 1) {
            int mid = (lo + hi) / 2;
            if (e2m1_code_value(mid) <= a) lo = mid; else hi = mid;
        }
        double dlo = a - e2m1_code_value(lo), dhi = e2m1_code_value(hi) - a;
        if (dlo < dhi) code = lo;
        else if (dhi < dlo) code = hi;
        else code = (lo & 1) ? hi : lo; /* tie: even mantissa */
    }
    return (uint8_t)(code | (neg << 3));
}

/* Second-level NVFP4 scale of a row (or matrix) from its largest
 * magnitude: g = amax / (6 * 448) in fp32, so that the largest block scale
 * is at most E4M3's 448 and the largest element at most E2M1's 6; an
 * all-zero (or underflowing) amax gives g = 1. */
static float nvfp4_global(float amax) {
    float g = amax / 2688.0f;
    return (amax > 0.0f && g > 0.0f) ? g : 1.0f;
}

/* NVFP4 quantisation of n values (n a multiple of 16) under the second-
 * level scale g.  Per block of 16: s = E4M3((amax_b / g) / 6) (fp32
 * divisions in that order, the E4M3 rounding to nearest-even and
 * saturating); the block's divisor d = value(s) * g (fp32); each element
 * v -> E2M1(v / d) (fp32 division, then the E2M1 rounding), or the signed
 * zero code when d is 0.  Codes are packed two per byte, element 2i in the
 * low nibble.  Dequantised: value(code) * value(s) * g. */
static void nvfp4_row(const float* v, int n, float g, uint8_t* q, uint8_t* s) {
    for (int b = 0; b < n / 16; ++b) {
        float amax = 0.0f;
        for (int i = 0; i < 16; ++i) {
            float a = fabsf(v[b * 16 + i]);
            if (a > amax) amax = a;
        }
        float sf = (amax / g) / 6.0f;
        uint8_t sb = e4m3_encode_rne_sat((double)sf);
        float d = (float)g_e4m3_all[sb] * g;
        s[b] = sb;
        for (int i = 0; i < 16; i += 2) {
            uint8_t c[2];
            for (int h = 0; h < 2; ++h) {
                float x = v[b * 16 + i + h];
                c[h] = d != 0.0f ? e2m1_encode_rne_sat((double)(x / d)) : (uint8_t)(signbit(x) ? 8 : 0);
            }
            q[(b * 16 + i) / 2] = (uint8_t)(c[0] | (c[1] << 4));
        }
    }
}

static float row_amax(const float* v, int64_t n) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(v[i]);
        if (a > amax) amax = a;
    }
    return amax;
}

/* ------------------------------------------------------------------ */
/* Public entry points (called through ctypes by the tests)           */
/* ------------------------------------------------------------------ */

int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

double oracle_e4m3_value(int code) { return e4m3_code_value(code & 255); }

/* MXFP8 quantisation of a row-major fp32 matrix [rows, cols] (values are
 * exact bf16 or fp32 numbers), blocks of 32 along each row.  cols must be a
 * multiple of 32.  q: [rows, cols] codes; s: [rows, cols/32] E8M0 bytes. */
int oracle_mxfp8_quantize(const float* in, int64_t rows, int64_t cols,
                          uint8_t* q, uint8_t* s) {
    if (!in || !q || !s || rows < 0 || cols <= 0 || (cols % 32) != 0) return ORACLE_EINVAL;
    build_tables();
    const int64_t nb = cols / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double v[32];
        for (int64_t b = 0; b < nb; ++b) {
            for (int i = 0; i < 32; ++i) v[i] = (double)in[r * cols + b * 32 + i];
            mxfp8_block(v, 32, q + r * cols + b * 32, s + r * nb + b);
        }
    }
    return ORACLE_OK;
}

/* Same, for a matrix given as bf16 bit patterns. */
int oracle_mxfp8_quantize_bf16(const uint16_t* in, int64_t rows, int64_t cols,
                               uint8_t* q, uint8_t* s) {
    if (!in || !q || !s || rows < 0 || cols <= 0 || (cols % 32) != 0) return ORACLE_EINVAL;
    build_tables();
    const int64_t nb = cols / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double v[32];
        for (int64_t b = 0; b < nb; ++b) {
            for (int i = 0; i < 32; ++i) v[i] = (double)bf16_bits_to_float(in[r * cols + b * 32 + i]);
            mxfp8_block(v, 32, q + r * cols + b * 32, s + r * nb + b);
        }
    }
    return ORACLE_OK;
}

/* Dequantise: out[r,c] = value(q[r,c]) * 2^(s[r,c/32]-127), in fp32 (exact
 * for every code/scale pair that a bf16 input can produce). */
int oracle_mxfp8_dequantize(const uint8_t* q, const uint8_t* s, int64_t rows, int64_t cols,
                            float* out) {
    if (!q || !s || !out || rows < 0 || cols <= 0 || (cols % 32) != 0) return ORACLE_EINVAL;
    build_tables();
    const int64_t nb = cols / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            out[r * cols + c] = (float)(g_e4m3_all[q[r * cols + c]] * g_pow2[s[r * nb + c / 32]]);
    return ORACLE_OK;
}

/* NVFP4 quantisation of a row-major fp32 matrix [rows, cols] (cols a
 * multiple of 16): codes [rows, cols/2], E4M3 block scales [rows, cols/16]
 * and the second-level scale: per row (per_row = 1, g_out[rows]) or one for
 * the whole matrix (per_row = 0, g_out[1]). */
int oracle_nvfp4_quantize(const float* in, int64_t rows, int64_t cols, int per_row,
                          uint8_t* q, uint8_t* s, float* g_out) {
    if (!in || !q || !s || !g_out || rows < 0 || cols <= 0 || (cols % 16)) return ORACLE_EINVAL;
    build_tables();
    float g_all = per_row ? 0.0f : nvfp4_global(row_amax(in, rows * cols));
    if (!per_row) g_out[0] = g_all;
    for (int64_t r = 0; r < rows; ++r) {
        float g = per_row ? nvfp4_global(row_amax(in + r * cols, cols)) : g_all;
        if (per_row) g_out[r] = g;
        nvfp4_row(in + r * cols, (int)cols, g, q + r * (cols / 2), s + r * (cols / 16));
    }
    return ORACLE_OK;
}

/* Same, for a matrix given as bf16 bit patterns. */
int oracle_nvfp4_quantize_bf16(const uint16_t* in, int64_t rows, int64_t cols, int per_row,
                               uint8_t* q, uint8_t* s, float* g_out) {
    if (!in || rows < 0 || cols <= 0) return ORACLE_EINVAL;
    float* f = (float*)malloc(sizeof(float) * (size_t)(rows * cols > 0 ? rows * cols : 1));
    if (!f) return ORACLE_ENOMEM;
    for (int64_t i = 0; i < rows * cols; ++i) f[i] = bf16_bits_to_float(in[i]);
    int rc = oracle_nvfp4_quantize(f, rows, cols, per_row, q, s, g_out);
    free(f);
    return rc;
}

/* Dequantise: out[r,c] = value(code) * value(s[r,c/16]) * g, in double
 * (exact: at most 2 + 4 + 24 significant bits). */
int oracle_nvfp4_dequantize(const uint8_t* q, const uint8_t* s, const float* g, int64_t rows, int64_t cols,
                            int per_row, double* out) {
    if (!q || !s || !g || !out || rows < 0 || cols <= 0 || (cols % 16)) return ORACLE_EINVAL;
    build_tables();
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            int code = (q[r * (cols / 2) + c / 2] >> ((c & 1) * 4)) & 15;
            out[r * cols + c] = e2m1_code_value(code) * g_e4m3_all[s[r * (cols / 16) + c / 16]] *
                                (double)g[per_row ? r : 0];
        }
    return ORACLE_OK;
}

/* Router: per token, top-k of the E logits by value (ties: lower id first),
 * probabilities = softmax over all E experts renormalised over the chosen k,
 * which equals exp(l_j - m) / sum_{i in topk} exp(l_i - m); evaluated in
 * double and rounded once to fp32.  Output ids ascending, probs matching. */
int oracle_route(const float* logits, int64_t T, int E, int k,
                 int32_t* ids, float* probs) {
    if (!logits || !ids || !probs || T < 0 || E <= 0 || E > 1024 || k <= 0 || k > E) return ORACLE_EINVAL;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const float* l = logits + t * E;
        int chosen_id[1024];
        char taken[1024];
        memset(taken, 0, (size_t)E);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e; /* strict: lower id wins ties */
            }
            taken[best] = 1;
            chosen_id[j] = best;
        }
        double m = (double)l[chosen_id[0]];
        double w[1024];
        double z = 0.0;
        for (int j = 0; j < k; ++j) {
            w[j] = exp((double)l[chosen_id[j]] - m);
            z += w[j];
        }
        /* canonical order: ascending expert id (insertion sort on k items) */
        for (int a = 1; a < k; ++a) {
            int id = chosen_id[a];
            double ww = w[a];
            int b = a - 1;
            while (b >= 0 && chosen_id[b] > id) {
                chosen_id[b + 1] = chosen_id[b];
                w[b + 1] = w[b];
                --b;
            }
            chosen_id[b + 1] = id;
            w[b + 1] = ww;
        }
        for (int j = 0; j < k; ++j) {
            ids[t * k + j] = chosen_id[j];
            probs[t * k + j] = (float)(w[j] / z);
        }
    }
    return ORACLE_OK;
}

/* Permute: counts per expert, exclusive prefix sum -> offsets[E+1]; route
 * (t, j) with expert e goes to row offsets[e] + (number of earlier tokens
 * routed to e).  perm[row] = t*k + j, inv[t*k + j] = row. */
int oracle_permute(const int32_t* ids, int64_t T, int E, int k,
                   int64_t* offsets, int32_t* perm, int32_t* inv) {
    if (!ids || !offsets || !perm || !inv || T < 0 || E <= 0 || k <= 0) return ORACLE_EINVAL;
    int64_t* seen = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    if (!seen) return ORACLE_ENOMEM;
    for (int e = 0; e <= E; ++e) offsets[e] = 0;
    for (int64_t i = 0; i < T * k; ++i) {
        int e = ids[i];
        if (e < 0 || e >= E) { free(seen); return ORACLE_EINVAL; }
        offsets[e + 1] += 1;
    }
    for (int e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
    for (int64_t t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int e = ids[t * k + j];
            int64_t row = offsets[e] + seen[e];
            seen[e] += 1;
            perm[row] = (int32_t)(t * k + j);
            inv[t * k + j] = (int32_t)row;
        }
    }
    free(seen);
    return ORACLE_OK;
}

static double silu_d(double z) { return z / (1.0 + exp(-z)); }

#define ORACLE_PROBS_IN_FC1 1
#define ORACLE_SQUARED_RELU 2

/* The fp32 activation value of one (route, f) from its double
 * pre-activations: clamped when clamp > 0, silu(g) * u (or relu(g)^2 for
 * squared-ReLU experts, u unused), scaled by the route's probability when
 * the probabilities are applied in FC1. */
static float swiglu_value(double g, double u, double clamp, int flags, float p) {
    if (clamp > 0.0) {
        g = g < -clamp ? -clamp : (g > clamp ? clamp : g);
        u = u < -clamp ? -clamp : (u > clamp ? clamp : u);
    }
    double h;
    if (flags & ORACLE_SQUARED_RELU) {
        const double r = g > 0.0 ? g : 0.0;
        h = r * r;
    } else {
        h = silu_d(g) * u;
    }
    if (flags & ORACLE_PROBS_IN_FC1) h *= (double)p;
    return (float)h;
}

/* out[i] = bf16(in[i]) with round-to-nearest-even, for a bf16 finalize. */
int oracle_round_bf16(const float* in, int64_t n, uint16_t* out) {
    if (!in || !out || n < 0) return ORACLE_EINVAL;
    for (int64_t i = 0; i < n; ++i) out[i] = float_to_bf16_bits_rne(in[i]);
    return ORACLE_OK;
}

/* Canonical order of one token's routes: ascending expert id, carrying the
 * probability with its id. */
static void sort_routes(const int32_t* ids_in, const float* p_in, int k, int* ids, float* p) {
    for (int j = 0; j < k; ++j) { ids[j] = ids_in[j]; p[j] = p_in[j]; }
    for (int a = 1; a < k; ++a) {
        int id = ids[a];
        float pp = p[a];
        int b = a - 1;
        while (b >= 0 && ids[b] > id) { ids[b + 1] = ids[b]; p[b + 1] = p[b]; --b; }
        ids[b + 1] = id;
        p[b + 1] = pp;
    }
}

/* bf16 forward for a list of tokens.
 *   x      [T, H]    bf16 bits          w_gate, w_up [E, F, H] bf16 bits
 *   ids    [T, k]    int32              w_down       [E, H, F] bf16 bits
 *   probs  [T, k]    fp32
 *   toks   [ntok]    token indices to evaluate
 *   out    [ntok, H] fp32
 *   h_out  [ntok, k, F] fp32 (nullable): the bf16-rounded SwiGLU row of each
 *          route, in canonical (ascending id) order.
 * Per route: g_f = sum_c Wg[e,f,c] x_c and u_f likewise (double);
 * h_f = bf16(fp32(silu(g_f) * u_f)); y_c = fp32(sum_f Wd[e,c,f] h_f);
 * out_c = fmaf(p_j, y_c, out_c) over j in ascending id, from 0.0f.
 * flags / clamp select the variants above (0, 0.0: the plain forward). */
int oracle_forward_bf16(const uint16_t* x, const int32_t* ids, const float* probs,
                        const uint16_t* w_gate, const uint16_t* w_up, const uint16_t* w_down,
                        int64_t T, int H, int F, int E, int k,
                        const int64_t* toks, int64_t ntok, float* out, float* h_out,
                        int flags, double clamp) {
    const int relu2 = (flags & ORACLE_SQUARED_RELU) != 0;
    if (!x || !ids || !probs || !w_gate || (!w_up && !relu2) || !w_down || !toks || !out) return ORACLE_EINVAL;
    if (H <= 0 || F <= 0 || E <= 0 || k <= 0 || k > 64 || ntok < 0) return ORACLE_EINVAL;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t i = 0; i < ntok; ++i) {
        int64_t t = toks[i];
        if (t < 0 || t >= T) { bad = 1; continue; }
        double* xd = (double*)malloc(sizeof(double) * (size_t)H);
        double* hd = (double*)malloc(sizeof(double) * (size_t)F);
        float* acc = out + i * H;
        int sid[64];
        float sp[64];
        if (!xd || !hd) { free(xd); free(hd); bad = 1; continue; }
        for (int c = 0; c < H; ++c) xd[c] = (double)bf16_bits_to_float(x[t * H + c]);
        for (int c = 0; c < H; ++c) acc[c] = 0.0f;
        sort_routes(ids + t * k, probs + t * k, k, sid, sp);
        for (int j = 0; j < k; ++j) {
            int e = sid[j];
            if (e < 0 || e >= E) { bad = 1; break; }
            const uint16_t* wg = w_gate + (int64_t)e * F * H;
            const uint16_t* wu = relu2 ? NULL : w_up + (int64_t)e * F * H;
            const uint16_t* wd = w_down + (int64_t)e * H * F;
            for (int f = 0; f < F; ++f) {
                double g = 0.0, u = 0.0;
                for (int c = 0; c < H; ++c) {
                    g += (double)bf16_bits_to_float(wg[(int64_t)f * H + c]) * xd[c];
                    if (!relu2) u += (double)bf16_bits_to_float(wu[(int64_t)f * H + c]) * xd[c];
                }
                float hf = swiglu_value(g, u, clamp, flags, sp[j]);
                float hb = bf16_bits_to_float(float_to_bf16_bits_rne(hf));
                hd[f] = (double)hb;
                if (h_out) h_out[(i * k + j) * F + f] = hb;
            }
            for (int c = 0; c < H; ++c) {
                double y = 0.0;
                for (int f = 0; f < F; ++f) y += (double)bf16_bits_to_float(wd[(int64_t)c * F + f]) * hd[f];
                acc[c] = (flags & ORACLE_PROBS_IN_FC1) ? acc[c] + (float)y : fmaf(sp[j], (float)y, acc[c]);
            }
        }
        free(xd);
        free(hd);
    }
    return bad ? ORACLE_EINVAL : ORACLE_OK;
}

/* MXFP8 forward for a list of tokens.  The weights arrive already quantised
 * (codes + E8M0 bytes, as oracle_mxfp8_quantize_bf16 makes them from the
 * bf16 weights):
 *   wg_q, wu_q [E, F, H] codes, wg_s, wu_s [E, F, H/32]  (blocks along H)
 *   wd_q       [E, H, F] codes, wd_s       [E, H, F/32]  (blocks along F)
 * x rows are quantised here from their bf16 values (blocks along H).  The
 * GEMMs use the dequantised operands exactly; h is formed as in the bf16
 * path up to its fp32 value, then quantised (blocks of 32 along F) and the
 * dequantised h enters the down GEMM.
 *   h_q_out [ntok, k, F] codes and h_s_out [ntok, k, F/32] (nullable),
 *   h_f32_out [ntok, k, F] pre-quantisation fp32 h (nullable).
 * flags / clamp select the variants above (0, 0.0: the plain forward). */
int oracle_forward_mxfp8(const uint16_t* x, const int32_t* ids, const float* probs,
                         const uint8_t* wg_q, const uint8_t* wg_s,
                         const uint8_t* wu_q, const uint8_t* wu_s,
                         const uint8_t* wd_q, const uint8_t* wd_s,
                         int64_t T, int H, int F, int E, int k,
                         const int64_t* toks, int64_t ntok, float* out,
                         uint8_t* h_q_out, uint8_t* h_s_out, float* h_f32_out, int flags, double clamp) {
    const int relu2 = (flags & ORACLE_SQUARED_RELU) != 0;
    if (!x || !ids || !probs || !wg_q || !wg_s || (!relu2 && (!wu_q || !wu_s)) || !wd_q || !wd_s || !toks || !out)
        return ORACLE_EINVAL;
    if (H <= 0 || F <= 0 || (H % 32) || (F % 32) || E <= 0 || k <= 0 || k > 64 || ntok < 0)
        return ORACLE_EINVAL;
    build_tables();
    const int nbh = H / 32, nbf = F / 32;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t i = 0; i < ntok; ++i) {
        int64_t t = toks[i];
        if (t < 0 || t >= T) { bad = 1; continue; }
        double* xv = (double*)malloc(sizeof(double) * (size_t)H);
        double* xd = (double*)malloc(sizeof(double) * (size_t)H);
        double* hv = (double*)malloc(sizeof(double) * (size_t)F);
        double* hd = (double*)malloc(sizeof(double) * (size_t)F);
        uint8_t* qb = (uint8_t*)malloc((size_t)(H > F ? H : F));
        float* acc = out + i * H;
        int sid[64];
        float sp[64];
        if (!xv || !xd || !hv || !hd || !qb) {
            free(xv); free(xd); free(hv); free(hd); free(qb);
            bad = 1;
            continue;
        }
        /* x: bf16 -> MXFP8 along H -> dequantised values */
        for (int c = 0; c < H; ++c) xv[c] = (double)bf16_bits_to_float(x[t * H + c]);
        for (int b = 0; b < nbh; ++b) {
            uint8_t sb;
            mxfp8_block(xv + b * 32, 32, qb + b * 32, &sb);
            for (int c = 0; c < 32; ++c) xd[b * 32 + c] = g_e4m3_all[qb[b * 32 + c]] * g_pow2[sb];
        }
        for (int c = 0; c < H; ++c) acc[c] = 0.0f;
        sort_routes(ids + t * k, probs + t * k, k, sid, sp);
        for (int j = 0; j < k; ++j) {
            int e = sid[j];
            if (e < 0 || e >= E) { bad = 1; break; }
            const uint8_t* gq = wg_q + (int64_t)e * F * H;
            const uint8_t* gs = wg_s + (int64_t)e * F * nbh;
            const uint8_t* uq = relu2 ? NULL : wu_q + (int64_t)e * F * H;
            const uint8_t* us = relu2 ? NULL : wu_s + (int64_t)e * F * nbh;
            const uint8_t* dq = wd_q + (int64_t)e * H * F;
            const uint8_t* ds = wd_s + (int64_t)e * H * nbf;
            for (int f = 0; f < F; ++f) {
                double g = 0.0, u = 0.0;
                for (int c = 0; c < H; ++c) {
                    double wgv = g_e4m3_all[gq[(int64_t)f * H + c]] * g_pow2[gs[(int64_t)f * nbh + c / 32]];
                    g += wgv * xd[c];
                    if (!relu2) {
                        double wuv = g_e4m3_all[uq[(int64_t)f * H + c]] * g_pow2[us[(int64_t)f * nbh + c / 32]];
                        u += wuv * xd[c];
                    }
                }
                float hf = swiglu_value(g, u, clamp, flags, sp[j]);
                hv[f] = (double)hf;
                if (h_f32_out) h_f32_out[(i * k + j) * F + f] = hf;
            }
            for (int b = 0; b < nbf; ++b) {
                uint8_t sb;
                mxfp8_block(hv + b * 32, 32, qb + b * 32, &sb);
                for (int c = 0; c < 32; ++c) hd[b * 32 + c] = g_e4m3_all[qb[b * 32 + c]] * g_pow2[sb];
                if (h_s_out) h_s_out[(i * k + j) * nbf + b] = sb;
            }
            if (h_q_out) memcpy(h_q_out + (i * k + j) * F, qb, (size_t)F);
            for (int c = 0; c < H; ++c) {
                double y = 0.0;
                for (int f = 0; f < F; ++f)
                    y += g_e4m3_all[dq[(int64_t)c * F + f]] * g_pow2[ds[(int64_t)c * nbf + f / 32]] * hd[f];
                acc[c] = (flags & ORACLE_PROBS_IN_FC1) ? acc[c] + (float)y : fmaf(sp[j], (float)y, acc[c]);
            }
        }
        free(xv); free(xd); free(hv); free(hd); free(qb);
    }
    return bad ? ORACLE_EINVAL : ORACLE_OK;
}

/* NVFP4 forward for a list of tokens (the per-token recipe above).  The
 * weights arrive quantised, as oracle_nvfp4_quantize makes them from the
 * bf16 weights with one second-level scale per expert matrix:
 *   w1_q [E, 2F, H/2], w1_s [E, 2F, H/16], g1 [E]: rows 0..F-1 the gate
 *       projection, F..2F-1 the up projection (one matrix, one scale);
 *       squared-ReLU experts (flags) have only the F gate rows;
 *   wd_q [E, H, F/2],  wd_s [E, H, F/16],  g2 [E].
 * x rows are quantised here from their bf16 values with a scale per token.
 * The GEMMs use the dequantised operands exactly; h is formed as in the
 * bf16 path up to its fp32 value, then quantised with a scale per route row
 * (blocks of 16 along F), and the dequantised h enters the down GEMM.
 *   h_q_out [ntok, k, F/2], h_s_out [ntok, k, F/16], h_g_out [ntok, k] and
 *   h_f32_out [ntok, k, F] (each nullable). */
int oracle_forward_nvfp4(const uint16_t* x, const int32_t* ids, const float* probs,
                         const uint8_t* w1_q, const uint8_t* w1_s, const float* g1,
                         const uint8_t* wd_q, const uint8_t* wd_s, const float* g2,
                         int64_t T, int H, int F, int E, int k,
                         const int64_t* toks, int64_t ntok, float* out,
                         uint8_t* h_q_out, uint8_t* h_s_out, float* h_g_out, float* h_f32_out, int flags,
                         double clamp) {
    const int relu2 = (flags & ORACLE_SQUARED_RELU) != 0;
    const int R1 = relu2 ? F : 2 * F;
    if (!x || !ids || !probs || !w1_q || !w1_s || !g1 || !wd_q || !wd_s || !g2 || !toks || !out)
        return ORACLE_EINVAL;
    if (H <= 0 || F <= 0 || (H % 16) || (F % 16) || E <= 0 || k <= 0 || k > 64 || ntok < 0)
        return ORACLE_EINVAL;
    build_tables();
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t i = 0; i < ntok; ++i) {
        int64_t t = toks[i];
        if (t < 0 || t >= T) { bad = 1; continue; }
        float* xf = (float*)malloc(sizeof(float) * (size_t)H);
        double* xd = (double*)malloc(sizeof(double) * (size_t)H);
        float* hf = (float*)malloc(sizeof(float) * (size_t)F);
        double* hd = (double*)malloc(sizeof(double) * (size_t)F);
        uint8_t* qb = (uint8_t*)malloc((size_t)(H > F ? H : F));
        uint8_t* sb = (uint8_t*)malloc((size_t)(H > F ? H : F) / 16);
        float* acc = out + i * H;
        int sid[64];
        float sp[64];
        if (!xf || !xd || !hf || !hd || !qb || !sb) {
            free(xf); free(xd); free(hf); free(hd); free(qb); free(sb);
            bad = 1;
            continue;
        }
        /* x: bf16 -> NVFP4 with this token's scale -> dequantised values */
        for (int c = 0; c < H; ++c) xf[c] = bf16_bits_to_float(x[t * H + c]);
        float gx = nvfp4_global(row_amax(xf, H));
        nvfp4_row(xf, H, gx, qb, sb);
        for (int c = 0; c < H; ++c)
            xd[c] = e2m1_code_value((qb[c / 2] >> ((c & 1) * 4)) & 15) * g_e4m3_all[sb[c / 16]] * (double)gx;
        for (int c = 0; c < H; ++c) acc[c] = 0.0f;
        sort_routes(ids + t * k, probs + t * k, k, sid, sp);
        for (int j = 0; j < k; ++j) {
            int e = sid[j];
            if (e < 0 || e >= E) { bad = 1; break; }
            const uint8_t* q1 = w1_q + (int64_t)e * R1 * (H / 2);
            const uint8_t* s1 = w1_s + (int64_t)e * R1 * (H / 16);
            const uint8_t* q2 = wd_q + (int64_t)e * H * (F / 2);
            const uint8_t* s2 = wd_s + (int64_t)e * H * (F / 16);
            for (int f = 0; f < F; ++f) {
                double gsum = 0.0, usum = 0.0;
                for (int c = 0; c < H; ++c) {
                    int64_t rg = f, ru = F + f;
                    double wg = e2m1_code_value((q1[rg * (H / 2) + c / 2] >> ((c & 1) * 4)) & 15) *
                                g_e4m3_all[s1[rg * (H / 16) + c / 16]] * (double)g1[e];
                    gsum += wg * xd[c];
                    if (!relu2) {
                        double wu = e2m1_code_value((q1[ru * (H / 2) + c / 2] >> ((c & 1) * 4)) & 15) *
                                    g_e4m3_all[s1[ru * (H / 16) + c / 16]] * (double)g1[e];
                        usum += wu * xd[c];
                    }
                }
                hf[f] = swiglu_value(gsum, usum, clamp, flags, sp[j]);
                if (h_f32_out) h_f32_out[(i * k + j) * F + f] = hf[f];
            }
            float gh = nvfp4_global(row_amax(hf, F));
            nvfp4_row(hf, F, gh, qb, sb);
            for (int f = 0; f < F; ++f)
                hd[f] = e2m1_code_value((qb[f / 2] >> ((f & 1) * 4)) & 15) * g_e4m3_all[sb[f / 16]] * (double)gh;
            if (h_q_out) memcpy(h_q_out + (i * k + j) * (F / 2), qb, (size_t)(F / 2));
            if (h_s_out) memcpy(h_s_out + (i * k + j) * (F / 16), sb, (size_t)(F / 16));
            if (h_g_out) h_g_out[i * k + j] = gh;
            for (int c = 0; c < H; ++c) {
                double y = 0.0;
                for (int f = 0; f < F; ++f)
                    y += e2m1_code_value((q2[(int64_t)c * (F / 2) + f / 2] >> ((f & 1) * 4)) & 15) *
                         g_e4m3_all[s2[(int64_t)c * (F / 16) + f / 16]] * (double)g2[e] * hd[f];
                acc[c] = (flags & ORACLE_PROBS_IN_FC1) ? acc[c] + (float)y : fmaf(sp[j], (float)y, acc[c]);
            }
        }
        free(xf); free(xd); free(hf); free(hd); free(qb); free(sb);
    }
    return bad ? ORACLE_EINVAL : ORACLE_OK;
}
