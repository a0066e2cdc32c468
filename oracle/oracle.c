/*
 * CPU oracle for fine-grained W4A8 linear-layer compute with the Integer-Scale
 * scheme.  TEST INFRASTRUCTURE ONLY: it is called by the tests, by the smoke
 * check and by the CPU-baseline leg of the benchmark, never by the product
 * path.  It shares no code, header or table with the CUDA library.
 *
 * Plain scalar loops, int64 accumulation, fp64 for every floating-point
 * result that no page fixes.  Where floating point decides an integer (a
 * quantized code), the decision is taken in IEEE fp32 with a true division,
 * the precision the CUDA kernels use, so that codes can be compared bit for bit.
 *
 * Sources (page title, section / equation):
 *  [Q]  "Quantization" notes, sections "量化公式" and "Symmetric Quantization":
 *       q = clip(round(x/s) + z, qmin, qmax); x_hat = s (q - z); symmetric:
 *       alpha = max|x|, s = alpha / qmax, z = 0, q in [-qmax, qmax], int8 qmax = 127.
 *  [Q-asym] same notes, "Asymmetric Quantization": the range [x_min, x_max]
 *       maps onto [qmin, qmax], s = (x_max - x_min) / (qmax - qmin),
 *       z = clip(round(qmin - x_min / s), qmin, qmax), q = clip(round(x / s) + z).
 *  [Q-mm] same notes, "矩阵乘法中的量化计算": with z = 0 on both operands the
 *       integer part of a quantized matmul is q_W q_X alone; with Z_W = 0 and an
 *       activation zero point it is (q_X - Z_X) q_W.
 *  [T34] "探秘Transformer系列之（34）量化基礎", §2.2.1 eqs. (1)-(2) and "Scale
 *       Quantization" (int8 symmetric range [-127, 127]); §2.3.3 "逐组量化"
 *       (one scale per group of K consecutive inputs of a weight column) and
 *       "逐通道量化 & 逐token量化" (one activation scale per token row).
 *  [IS] "Integer Scale: A Free Lunch for Faster Fine-grained Quantization of
 *       LLMs" summary, §3.2 / Fig. 3(b) (float group scales, one I32->F32
 *       conversion per group result), §4 / Fig. 3(c) (integer scales
 *       round(s_g * alpha), integer accumulation, one final rescale by
 *       s_a / alpha), §4 amplifier search, §5.1 Table 1 (group 128, symmetric,
 *       amplifier 1024).
 *  [X4] "极致量化", "其他子4位整数格式" and "数据打包" (low-bit values packed
 *       into a standard integer type).
 *
 * Readings where the pages are silent (all listed in the design notes):
 *  - round() is round-half-to-even (C rint() in the default rounding mode);
 *  - an all-zero row or group gets scale 0 and codes 0;
 *  - int4 weights are symmetric with qmax = 7 (range [-7, 7]);
 *  - nibble packing, K-contiguous per column n: every 8 codes along K fill
 *    one 32-bit word (4 bytes); code i of the 8 sits in byte i mod 4, in the
 *    low nibble for i < 4 and the high nibble for i >= 4 (two's complement);
 *  - the GEMM accumulates in int32: every accumulator of a call must lie in
 *    (-2^31, 2^31); the accumulating functions count those that do not;
 *  - the amplifier search ignores zero scales, and returns 1 when the
 *    smallest scale is already >= 1.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ---- [Q] symmetric scale and one code ----------------------------------- */

/* s = alpha / qmax with alpha = max|x|, computed in IEEE fp32 ([Q] Symmetric). */
static float symmetric_scale(float absmax, int32_t qmax) {
    volatile float a = absmax; /* keep the division a single fp32 operation */
    return a / (float)qmax;
}

/* q = clip(round(x / s), -qmax, qmax), z = 0 ([Q] 量化公式, [T34] eq. (1)). */
static int32_t symmetric_code(float x, float s, int32_t qmax) {
    if (s == 0.0f) return 0;
    volatile float t = x / s; /* one IEEE fp32 division */
    double r = rint((double)t); /* round half to even */
    if (r > qmax) r = qmax;
    if (r < -qmax) r = -qmax;
    return (int32_t)r;
}

/* Per-row (per-token) symmetric quantization of x [rows, cols] ([T34]
 * 逐token量化; [IS] §5.4 per-token 8-bit activations). */
void oracle_quantize_rows(const float* x, int64_t rows, int64_t cols, int32_t qmax,
                          int8_t* q, float* s) {
    for (int64_t m = 0; m < rows; ++m) {
        const float* xr = x + m * cols;
        float a = 0.0f;
        for (int64_t k = 0; k < cols; ++k) {
            float v = fabsf(xr[k]);
            if (v > a) a = v;
        }
        float sm = (a == 0.0f) ? 0.0f : symmetric_scale(a, qmax);
        s[m] = sm;
        for (int64_t k = 0; k < cols; ++k) q[m * cols + k] = (int8_t)symmetric_code(xr[k], sm, qmax);
    }
}

/* Per-row asymmetric quantization of x [rows, cols] ([Q-asym]; one scale and
 * one zero point per token row as in [T34] 逐token量化).  Each step is one IEEE
 * fp32 operation: d = x_max - x_min, s = d / (qmax - qmin), t = x_min / s,
 * u = qmin - t, z = clip(rint(u)), and per element q = clip(rint(x / s) + z).
 * Readings where the notes are silent: round() is half to even; a constant
 * row (x_max = x_min) has an empty range, which is widened to include zero
 * (so a constant c is reconstructed to within the rounding of s); a row whose
 * scale is 0 (all zeros, or a range too small for an fp32 scale) gets z = 0
 * and codes 0.  The clip of z acts only when the range excludes zero. */
void oracle_quantize_rows_asym(const float* x, int64_t rows, int64_t cols, int32_t qmin, int32_t qmax,
                               int8_t* q, float* s, int32_t* z) {
    for (int64_t m = 0; m < rows; ++m) {
        const float* xr = x + m * cols;
        float lo = xr[0], hi = xr[0];
        for (int64_t k = 1; k < cols; ++k) {
            if (xr[k] < lo) lo = xr[k];
            if (xr[k] > hi) hi = xr[k];
        }
        if (hi == lo) {
            if (lo > 0.0f) lo = 0.0f;
            if (hi < 0.0f) hi = 0.0f;
        }
        volatile float d = hi - lo;
        volatile float sm = d / (float)(qmax - qmin);
        s[m] = sm;
        if (sm == 0.0f) {
            z[m] = 0;
            for (int64_t k = 0; k < cols; ++k) q[m * cols + k] = 0;
            continue;
        }
        volatile float t = lo / sm;
        volatile float u = (float)qmin - t;
        double zr = rint((double)u);
        if (zr < qmin) zr = qmin;
        if (zr > qmax) zr = qmax;
        const int32_t zm = (int32_t)zr;
        z[m] = zm;
        for (int64_t k = 0; k < cols; ++k) {
            volatile float v = xr[k] / sm;
            double r = rint((double)v) + (double)zm;
            if (r < qmin) r = qmin;
            if (r > qmax) r = qmax;
            q[m * cols + k] = (int8_t)r;
        }
    }
}

/* Per-group symmetric quantization of w [K, N] (row-major): one scale per
 * (group of `group` consecutive k, column n) ([T34] 逐组量化; [IS] Fig. 3(a);
 * [IS] §4 counts 131072 such scales for a 4096x4096 layer in groups of 128).
 * Codes q [K, N], scales s_g [K/group, N]. */
void oracle_quantize_groups(const float* w, int64_t K, int64_t N, int64_t group, int32_t qmax,
                            int8_t* q, float* s_g) {
    int64_t G = K / group;
    for (int64_t g = 0; g < G; ++g) {
        for (int64_t n = 0; n < N; ++n) {
            float a = 0.0f;
            for (int64_t k = g * group; k < (g + 1) * group; ++k) {
                float v = fabsf(w[k * N + n]);
                if (v > a) a = v;
            }
            float sg = (a == 0.0f) ? 0.0f : symmetric_scale(a, qmax);
            s_g[g * N + n] = sg;
            for (int64_t k = g * group; k < (g + 1) * group; ++k)
                q[k * N + n] = (int8_t)symmetric_code(w[k * N + n], sg, qmax);
        }
    }
}

/* Per-group quantization over the full signed 4-bit range [-8, 7] ([X4]
 * 其他子4位整数格式: a signed N-bit integer holds [-2^(N-1), 2^(N-1) - 1]).
 * Reading: the scale divides the group's max |w| by 8, so the group's most
 * negative extreme is code -8 and a positive extreme clips to 7:
 * s_g = fl32(max|w| / 8), q = clip(rne(fl32(w / s_g)), -8, 7). */
void oracle_quantize_groups_full_range(const float* w, int64_t K, int64_t N, int64_t group, int8_t* q,
                                       float* s_g) {
    int64_t G = K / group;
    for (int64_t g = 0; g < G; ++g) {
        for (int64_t n = 0; n < N; ++n) {
            float a = 0.0f;
            for (int64_t k = g * group; k < (g + 1) * group; ++k) {
                float v = fabsf(w[k * N + n]);
                if (v > a) a = v;
            }
            float sg = (a == 0.0f) ? 0.0f : symmetric_scale(a, 8);
            s_g[g * N + n] = sg;
            for (int64_t k = g * group; k < (g + 1) * group; ++k) {
                int32_t c = 0;
                if (sg != 0.0f) {
                    volatile float t = w[k * N + n] / sg; /* one IEEE fp32 division */
                    double r = rint((double)t);          /* round half to even */
                    if (r > 7) r = 7;
                    if (r < -8) r = -8;
                    c = (int32_t)r;
                }
                q[k * N + n] = (int8_t)c;
            }
        }
    }
}

/* ---- [X4] nibble packing -------------------------------------------------- */

/* Layout (a reading: the pages only say that several low-bit values share one
 * standard integer).  Along K, every 8 codes fill one 32-bit word, 4 bytes:
 * code i of the 8 (k = 8b + i) sits in byte 4b + (i mod 4), in the low nibble
 * for i < 4 and the high nibble for i >= 4, as a two's-complement nibble.
 * K must be a multiple of 8. */
static int64_t packed_byte(int64_t k) { return (k >> 3) * 4 + (k & 3); }
static int packed_shift(int64_t k) { return (int)((k >> 2) & 1) * 4; }

void oracle_pack_int4(const int8_t* q, int64_t K, int64_t N, uint8_t* packed) {
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < K / 2; ++j) packed[n * (K / 2) + j] = 0;
        for (int64_t k = 0; k < K; ++k) {
            unsigned nib = (unsigned)(uint8_t)q[k * N + n] & 0xFu;
            packed[n * (K / 2) + packed_byte(k)] |= (uint8_t)(nib << packed_shift(k));
        }
    }
}

/* Two's-complement nibble back to a signed value. */
static int32_t nibble_value(unsigned nib) { return (nib & 0x8u) ? (int32_t)nib - 16 : (int32_t)nib; }

void oracle_unpack_int4(const uint8_t* packed, int64_t K, int64_t N, int8_t* q) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t b = packed[n * (K / 2) + packed_byte(k)];
            q[k * N + n] = (int8_t)nibble_value((b >> packed_shift(k)) & 0xFu);
        }
}

/* ---- [IS] §4 amplifier search --------------------------------------------- */

/* Start from the smallest scale of the layer and double the amplifier until
 * the amplified smallest scale reaches 1; the amplifier is that power of two.
 * Zero scales are left out (an empty group has nothing to amplify).  Returns
 * the amplifier, 1 when every scale is already >= 1 or no scale is positive,
 * and -1 when no power of two up to 2^30 is enough. */
int32_t oracle_amplifier_search(const float* scales, int64_t count) {
    float smin = 0.0f;
    int have = 0;
    for (int64_t i = 0; i < count; ++i) {
        float v = scales[i];
        if (v > 0.0f && (!have || v < smin)) {
            smin = v;
            have = 1;
        }
    }
    if (!have) return 1;
    double amplifier = 1.0;
    int shifts = 0;
    while ((double)smin * amplifier < 1.0) {
        amplifier *= 2.0;
        ++shifts;
        if (shifts > 30) return -1;
    }
    return (int32_t)amplifier;
}

/* Integer scales S = round(s_g * alpha) ([IS] §4, Fig. 3(c)).  The product is
 * exact (alpha is a power of two); rounding is half to even.  Returned as
 * int32 so that values beyond int16 stay visible to the caller. */
void oracle_integer_scales(const float* s_g, int64_t count, int32_t alpha, int32_t* S) {
    for (int64_t i = 0; i < count; ++i) S[i] = (int32_t)rint((double)s_g[i] * (double)alpha);
}

/* ---- [IS] Fig. 3(c): group integer GEMM + integer-scale accumulation ------ */

/* 1 when an accumulator leaves the int32 range the GPU accumulates in
 * ([IS] §4: the amplifier is kept at 1024 to stay clear of overflow). */
static int32_t outside_int32(int64_t v) { return v >= ((int64_t)1 << 31) || v <= -((int64_t)1 << 31); }

/* acc[m,n] = sum_g S[g,n] * P_g[m,n],  P_g[m,n] = sum_{k in g} qx[m,k] qw[k,n]
 * qx [M,K], qw [K,N] codes, S [G,N]; everything in int64.  Returns how many
 * accumulators lie outside int32 (0 for a valid input). */
int64_t oracle_intscale_acc(const int8_t* qx, const int8_t* qw, const int32_t* S, int64_t M,
                            int64_t N, int64_t K, int64_t group, int64_t* acc) {
    int64_t G = K / group, bad = 0;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t total = 0;
            for (int64_t g = 0; g < G; ++g) {
                int64_t p = 0;
                for (int64_t k = g * group; k < (g + 1) * group; ++k)
                    p += (int64_t)qx[m * K + k] * (int64_t)qw[k * N + n];
                total += (int64_t)S[g * N + n] * p;
            }
            acc[m * N + n] = total;
            bad += outside_int32(total);
        }
    return bad;
}

/* The same integer reached the other way round: first the integer weight
 * W_int[k,n] = S[g(k),n] * qw[k,n], then one dense integer matmul. */
void oracle_intscale_acc_expanded(const int8_t* qx, const int8_t* qw, const int32_t* S,
                                  int64_t M, int64_t N, int64_t K, int64_t group, int64_t* acc) {
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t total = 0;
            for (int64_t k = 0; k < K; ++k) {
                int64_t w_int = (int64_t)S[(k / group) * N + n] * (int64_t)qw[k * N + n];
                total += (int64_t)qx[m * K + k] * w_int;
            }
            acc[m * N + n] = total;
        }
}

/* Group-wise accumulators at selected output positions (m_i, n_i) only. */
int64_t oracle_intscale_acc_at(const int8_t* qx, const int8_t* qw, const int32_t* S, int64_t M,
                               int64_t N, int64_t K, int64_t group, const int64_t* ms,
                               const int64_t* ns, int64_t count, int64_t* acc) {
    (void)M;
    int64_t G = K / group, bad = 0;
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = ms[i], n = ns[i];
        int64_t total = 0;
        for (int64_t g = 0; g < G; ++g) {
            int64_t p = 0;
            for (int64_t k = g * group; k < (g + 1) * group; ++k)
                p += (int64_t)qx[m * K + k] * (int64_t)qw[k * N + n];
            total += (int64_t)S[g * N + n] * p;
        }
        acc[i] = total;
        bad += outside_int32(total);
    }
    return bad;
}

/* Integer-scale accumulation with an asymmetric activation ([Q-mm] with
 * Z_W = 0 and Z_X = z[m]; [IS] §4 integer group scales):
 * acc[m,n] = sum_g S[g,n] * sum_{k in g} (qx[m,k] - z[m]) * qw[k,n].
 * The final rescale is the same as the symmetric one, acc * s_a[m] / alpha. */
int64_t oracle_intscale_acc_asym(const int8_t* qx, const int32_t* z, const int8_t* qw, const int32_t* S,
                                 int64_t M, int64_t N, int64_t K, int64_t group, int64_t* acc) {
    int64_t G = K / group, bad = 0;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t total = 0;
            for (int64_t g = 0; g < G; ++g) {
                int64_t p = 0;
                for (int64_t k = g * group; k < (g + 1) * group; ++k)
                    p += ((int64_t)qx[m * K + k] - (int64_t)z[m]) * (int64_t)qw[k * N + n];
                total += (int64_t)S[g * N + n] * p;
            }
            acc[m * N + n] = total;
            bad += outside_int32(total);
        }
    return bad;
}

/* Final rescale, once per output: y = acc * s_a[m] / alpha, in fp64 ([IS] §4). */
void oracle_intscale_output(const int64_t* acc, const float* s_a, int32_t alpha, int64_t M,
                            int64_t N, double* y) {
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            y[m * N + n] = (double)acc[m * N + n] * (double)s_a[m] / (double)alpha;
}

/* ---- [IS] §3.2 / Fig. 3(b): float-scale comparison path ------------------- */

/* y[m,n] = s_a[m] * sum_g s_g[g,n] * float(P_g[m,n]), in fp64. */
void oracle_floatscale(const int8_t* qx, const float* s_a, const int8_t* qw, const float* s_g,
                       int64_t M, int64_t N, int64_t K, int64_t group, double* y) {
    int64_t G = K / group;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double total = 0.0;
            for (int64_t g = 0; g < G; ++g) {
                int64_t p = 0;
                for (int64_t k = g * group; k < (g + 1) * group; ++k)
                    p += (int64_t)qx[m * K + k] * (int64_t)qw[k * N + n];
                total += (double)s_g[g * N + n] * (double)p;
            }
            y[m * N + n] = (double)s_a[m] * total;
        }
}

void oracle_floatscale_at(const int8_t* qx, const float* s_a, const int8_t* qw, const float* s_g,
                          int64_t M, int64_t N, int64_t K, int64_t group, const int64_t* ms,
                          const int64_t* ns, int64_t count, double* y) {
    (void)M;
    int64_t G = K / group;
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = ms[i], n = ns[i];
        double total = 0.0;
        for (int64_t g = 0; g < G; ++g) {
            int64_t p = 0;
            for (int64_t k = g * group; k < (g + 1) * group; ++k)
                p += (int64_t)qx[m * K + k] * (int64_t)qw[k * N + n];
            total += (double)s_g[g * N + n] * (double)p;
        }
        y[i] = (double)s_a[m] * total;
    }
}

/* ---- [IS] §4, Fig. 4(a)/(c): amplifier analysis ------------------------- */

/* For each amplifier alphas[i]: the mean squared difference between the
 * weights dequantized with the integer scales and with the float scales,
 * mean over (k, n) of (q[k,n] * (S[g,n] / alpha - s_g[g,n]))^2 with
 * S = rne(s_g * alpha) as in oracle_integer_scales (Fig. 4(c)), and the bits
 * the largest S needs as an unsigned integer (Fig. 4(a)).  fp64 throughout. */
void oracle_alpha_sweep(const int8_t* q, const float* s_g, int64_t K, int64_t N, int64_t group,
                        const int32_t* alphas, int64_t n_alpha, double* mse, int32_t* max_bits) {
    int64_t G = K / group;
    for (int64_t i = 0; i < n_alpha; ++i) {
        double a = (double)alphas[i], sum = 0.0, smax = 0.0;
        for (int64_t g = 0; g < G; ++g)
            for (int64_t n = 0; n < N; ++n) {
                double sf = (double)s_g[g * N + n];
                double S = rint(sf * a);
                double d = S / a - sf;
                if (S > smax) smax = S;
                for (int64_t k = g * group; k < (g + 1) * group; ++k) {
                    double e = (double)q[k * N + n] * d;
                    sum += e * e;
                }
            }
        mse[i] = sum / ((double)K * (double)N);
        int32_t bits = 0;
        while (bits < 62 && (double)((int64_t)1 << bits) <= smax) ++bits;  /* smallest b with smax < 2^b */
        max_bits[i] = bits;
    }
}

/* ---- worst-case int32 bound ----------------------------------------------- */

/* max over columns n of sum_g |S[g,n]|, the factor that multiplies
 * max|qx| * max|qw| * group in the bound on |acc|. */
int64_t oracle_scale_colsum_max(const int32_t* S, int64_t G, int64_t N) {
    int64_t best = 0;
    for (int64_t n = 0; n < N; ++n) {
        int64_t t = 0;
        for (int64_t g = 0; g < G; ++g) t += S[g * N + n] < 0 ? -(int64_t)S[g * N + n] : S[g * N + n];
        if (t > best) best = t;
    }
    return best;
}
