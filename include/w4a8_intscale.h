/*
 * w4a8_intscale.h -- C ABI of the B200 (sm_100a) W4A8 Integer-Scale library.
 *
 * Fine-grained W4A8 linear-layer compute:
 *   y[m,n] = s_a[m]/alpha * sum_g S[g,n] * sum_{k in g} q_x[m,k] q_w[k,n]
 * with per-token symmetric int8 activations (q_x, s_a), per-group symmetric
 * int4 weights (q_w, float group scales s_g), and integer group scales
 * S = round(s_g * alpha) for a power-of-two amplifier alpha.
 *
 * Sources, by page and section:
 *  - "Quantization" notes, 量化公式 / Symmetric Quantization: q = clip(round(x/s)
 *    + z, qmin, qmax), s = max|x| / qmax, z = 0, int8 range [-127, 127];
 *    矩阵乘法中的量化计算: with z = 0 the integer part of a quantized matmul is
 *    q_W q_X alone.
 *  - 探秘Transformer系列之（34）量化基礎 §2.3.3: per-token activation scales,
 *    per-group weight scales (逐组量化).
 *  - "Integer Scale: A Free Lunch for Faster Fine-grained Quantization of LLMs"
 *    (summary): Fig. 3(a) shapes X [M,K], W [K,N]; §3.2 / Fig. 3(b) float-scale
 *    path (one I32->F32 conversion and float multiply per group result);
 *    §4 / Fig. 3(c) integer scales, integer accumulation, one rescale by
 *    s_a/alpha; §4 amplifier search; §5.1 Table 1 group 128, symmetric,
 *    amplifier 1024.
 *  - 极致量化, 数据打包: several int4 values stored in one byte.
 *
 * Conventions for every entry point:
 *  - Device pointers are caller-owned (any allocator); the library allocates
 *    no device memory.  Host pointers are named *_host.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Calls are asynchronous on it unless stated "synchronous".
 *  - Arguments are validated on the host before any launch; an error return
 *    means nothing was launched.  No C++ exception crosses the ABI.
 *  - Kernels bound every wait; a wait that runs out (about one second) makes
 *    the kernel return early and records W4A8_ERR_TIMEOUT in a device status
 *    word that w4a8_device_status() reads.  The tcgen05 GEMM kernels also
 *    record W4A8_ERR_ALIGN there, and return at once, if the device's
 *    dynamic shared memory does not start 1024-byte aligned (their layout
 *    needs it; not seen on B200).
 *  - The GEMMs run a persistent grid of at most one CTA per resident slot
 *    (SMs x CTAs per SM) and split the (tile, group) steps into one range per
 *    CTA.  A tile cut by two ranges is finished by one of its CTAs, which
 *    waits for the others' partial sums: this assumes that every CTA of the
 *    grid becomes resident.  A kernel on another stream that holds SMs for
 *    long can delay a call by up to the wait limit, after which it fails with
 *    W4A8_ERR_TIMEOUT instead of waiting forever.
 *  - Layouts are row-major.  All device pointers must be 16-byte aligned.
 *  - Readings where the pages are silent: round() is round half to even;
 *    an all-zero row or group gets scale 0 and codes 0; int4 codes are
 *    symmetric in [-7, 7]; inputs must be finite.
 */
#ifndef W4A8_INTSCALE_H
#define W4A8_INTSCALE_H

#include <stdint.h>

#if defined(__GNUC__)
#define W4A8_API __attribute__((visibility("default")))
#else
#define W4A8_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    W4A8_OK = 0,
    W4A8_ERR_INVALID_ARG = 1,    /* null pointer, bad enum, alpha not a power of two */
    W4A8_ERR_SHAPE = 2,          /* M/N/K/group outside what the kernels accept */
    W4A8_ERR_ALIGN = 3,          /* pointer or leading dimension not 16-byte aligned */
    W4A8_ERR_DTYPE = 4,          /* dtype not supported for this argument */
    W4A8_ERR_OVERFLOW_BOUND = 5, /* 127*7*group*max_n sum_g|S[g,n]| >= 2^31 */
    W4A8_ERR_SCALE_RANGE = 6,    /* S would exceed int16, or alpha > 2^30 needed */
    W4A8_ERR_CUDA = 7,           /* a CUDA runtime call failed */
    W4A8_ERR_TIMEOUT = 8,        /* a kernel wait ran out (device status only) */
    W4A8_ERR_WORKSPACE = 9       /* workspace missing or too small */
} w4a8_status;

typedef enum {
    W4A8_F32 = 0,
    W4A8_F16 = 1,
    W4A8_BF16 = 2,
    W4A8_I32 = 3 /* raw int32 accumulators (integer-scale GEMM only) */
} w4a8_dtype;

/* Human-readable name of a status code (static string). */
W4A8_API const char* w4a8_status_string(int32_t status);

/*
 * Per-token symmetric int8 activation quantization.
 * ("Quantization" notes, Symmetric Quantization; 探秘Transformer系列之（34）
 *  §2.3.3 逐token量化; Integer Scale summary §5.4 per-token 8-bit activations.)
 *   s_a[m] = fl32(max_k |x[m,k]| / 127)
 *   q_x[m,k] = clamp(rne(fl32(x[m,k] / s_a[m])), -127, 127)   (0 when s_a[m] = 0)
 * x       device, [M, ldx] of x_dtype (W4A8_F32 or W4A8_BF16); row m starts at x + m*ldx
 * M, K    M >= 0 (M = 0 is a no-op), K > 0 and K % 16 == 0; ldx >= K, ldx*sizeof(x) % 16 == 0
 * q_x     device, [M, K] int8, written
 * s_a     device, [M] float32, written
 * Errors: W4A8_ERR_DTYPE, W4A8_ERR_SHAPE as above; W4A8_ERR_INVALID_ARG for a NULL
 * pointer; W4A8_ERR_ALIGN unless x and q_x are 16-byte and s_a 4-byte aligned.
 */
W4A8_API w4a8_status quantize_act_per_token(const void* x, int32_t x_dtype, int64_t M, int64_t K, int64_t ldx,
                                   int8_t* q_x, float* s_a, void* stream);

/*
 * Per-token quantization in routed order, for the grouped expert call: row i
 * of the output holds the codes and the scale of token row_index[i], the same
 * bit for bit as quantize_act_per_token gives that token.  A mixture-of-experts
 * layer routes every token to top_k experts; with the routed rows laid out
 * expert by expert, the grouped call reads each tile's rows as one block.
 * (Integer Scale summary §5.3: the method applied to Mixtral 8x7B.)
 * x, x_dtype, K, ldx   as quantize_act_per_token, T token rows
 * row_index  device, [R] int32, 4-byte aligned: the token of each routed row.
 *            A token outside [0, T) gives that row zero codes and scale and sets
 *            W4A8_ERR_INVALID_ARG in the device status word
 * q_r, s_r   device, [R, K] int8 (16-byte aligned) and [R] float32 (4-byte)
 * Errors as quantize_act_per_token; R < 0 or T < 1 (with R > 0) is W4A8_ERR_SHAPE.
 */
W4A8_API w4a8_status quantize_act_routed(const void* x, int32_t x_dtype, int64_t T, int64_t K, int64_t ldx,
                                         const int32_t* row_index, int64_t R, int8_t* q_r, float* s_r,
                                         void* stream);

/*
 * Per-token asymmetric int8 activation quantization.
 * ("Quantization" notes, Asymmetric Quantization: the range [x_min, x_max]
 *  maps onto [q_min, q_max] = [-128, 127]; 探秘Transformer系列之（34）§2.3.3
 *  逐token量化.)  Every step is one IEEE fp32 operation:
 *   lo, hi  = min_k x[m,k], max_k x[m,k]; if lo == hi the range is widened to
 *             include zero (lo = min(lo, 0), hi = max(hi, 0))
 *   s_a[m]  = fl32(fl32(hi - lo) / 255)
 *   z_a[m]  = clamp(rne(fl32(-128 - fl32(lo / s_a[m]))), -128, 127)
 *   q_x[m,k] = clamp(rne(fl32(x[m,k] / s_a[m])) + z_a[m], -128, 127)
 *   (s_a[m] = 0: z_a[m] = 0 and the row's codes are 0)
 *   dequantized: x[m,k] ~ s_a[m] * (q_x[m,k] - z_a[m])
 * x, M, K, ldx as quantize_act_per_token (finite values)
 * q_x     device, [M, K] int8, written
 * s_a     device, [M] float32, written
 * z_a     device, [M] int32, written
 * Errors as quantize_act_per_token; z_a must be 4-byte aligned (W4A8_ERR_ALIGN).
 */
W4A8_API w4a8_status quantize_act_per_token_asym(const void* x, int32_t x_dtype, int64_t M, int64_t K, int64_t ldx,
                                                 int8_t* q_x, float* s_a, int32_t* z_a, void* stream);

/*
 * Amplifier search over a set of float group scales (synchronous).
 * (Integer Scale summary §4 heuristic search.)  alpha is the smallest power
 * of two 2^j, j >= 0, with s_min * alpha >= 1, s_min the smallest POSITIVE
 * scale; 1 when no scale is positive or s_min >= 1.
 * scales     device, [count] float32
 * workspace  device, >= W4A8_PACK_WORKSPACE_BYTES bytes, contents scratch
 * alpha_host host, written
 * Returns W4A8_ERR_SCALE_RANGE when alpha would exceed 2^30.
 */
#define W4A8_PACK_WORKSPACE_BYTES (1 << 20)
W4A8_API w4a8_status w4a8_amplifier_search(const float* scales, int64_t count, void* workspace,
                                  int32_t* alpha_host, void* stream);

/*
 * Per-group symmetric int4 weight quantization, nibble packing, amplifier and
 * integer scales (synchronous: it waits for the stream once or twice).
 * (探秘Transformer系列之（34）§2.3.3 逐组量化; Integer Scale summary Fig. 3(a),
 *  §4; 极致量化 数据打包.)
 *   s_g[g,n]  = fl32(max_{k in g} |w[k,n]| / 7)
 *   q_w[k,n]  = clamp(rne(fl32(w[k,n] / s_g[g(k),n])), -7, 7)
 *   w_packed[n, 4b + i] = (q_w[8b+i,n] & 0xF) | (q_w[8b+4+i,n] & 0xF) << 4   (i = 0..3):
 *               each 32-bit word holds 8 consecutive codes along K, code j in
 *               byte j mod 4, low nibble for j < 4, high nibble for j >= 4
 *   alpha     = alpha_in if alpha_in > 0 (must be a power of two <= 2^30),
 *               else the amplifier search over this layer's s_g
 *   S[g,n]    = rne(s_g[g,n] * alpha)
 * w          device, [K, N] float32
 * K, N       K % group == 0, N % 8 == 0, N > 0
 * group      even, group % 32 == 0 (128 in the method)
 * w_packed   device, [N, K/2] uint8, written; may be NULL together with S to
 *            compute s_g only (alpha_out and colsum_max_host are then untouched)
 * s_g        device, [K/group, N] float32, written
 * S          device, [K/group, N] int16, written (or NULL, see w_packed)
 * alpha_out_host      host int32, written: the alpha used
 * colsum_max_host     host int64, written (may be NULL): max_n sum_g |S[g,n]|
 * workspace  device, >= W4A8_PACK_WORKSPACE_BYTES bytes, contents scratch
 * Errors: W4A8_ERR_SCALE_RANGE if max S > 32767; W4A8_ERR_OVERFLOW_BOUND if
 * 127*7*group*colsum_max >= 2^31 (outputs are written in both cases).
 */
W4A8_API w4a8_status pack_w4_groupwise(const float* w, int64_t K, int64_t N, int32_t group, int32_t alpha_in,
                              uint8_t* w_packed, float* s_g, int16_t* S, int32_t* alpha_out_host,
                              int64_t* colsum_max_host, void* workspace, void* stream);

/*
 * pack_w4_groupwise with a choice of code range (极致量化 其他子4位整数格式:
 * a signed N-bit integer holds [-2^(N-1), 2^(N-1) - 1]).
 *   qmin = -7: s_g = max|w| / 7, codes clamp(rne(w / s_g), -7, 7)
 *              (what pack_w4_groupwise does);
 *   qmin = -8: s_g = max|w| / 8, codes clamp(rne(w / s_g), -8, 7): the full
 *              two's-complement range; a group's positive extreme clips to 7.
 * The overflow bound is then 127*8*group*colsum_max < 2^31.  The packed
 * layout, alpha and S are as above; the GEMMs accept either range.
 * Errors: as pack_w4_groupwise; W4A8_ERR_INVALID_ARG for any other qmin.
 */
W4A8_API w4a8_status pack_w4_groupwise_range(const float* w, int64_t K, int64_t N, int32_t group, int32_t alpha_in,
                                    int32_t qmin, uint8_t* w_packed, float* s_g, int16_t* S,
                                    int32_t* alpha_out_host, int64_t* colsum_max_host, void* workspace,
                                    void* stream);

/*
 * Fine-grained W8A8 weights (the pages' W8A8 configurations, Integer Scale
 * summary §5, with the same integer group scales): per-group symmetric 8-bit
 * weight codes, amplifier and integer scales (synchronous like
 * pack_w4_groupwise).
 *   s_g[g,n]  = fl32(max_{k in g} |w[k,n]| / 127)
 *   q_w[k,n]  = clamp(rne(fl32(w[k,n] / s_g[g(k),n])), -127, 127)
 *   w8[n, k]  = q_w[k,n]        (int8, K-contiguous per output column)
 *   alpha, S  as in pack_w4_groupwise
 * w          device, [K, N] float32
 * K, N       K % group == 0, N % 8 == 0, N > 0; group % 32 == 0
 * w8         device, [N, K] int8, written
 * s_g        device, [K/group, N] float32, written
 * S          device, [K/group, N] int16, written
 * alpha_out_host, colsum_max_host, workspace: as in pack_w4_groupwise
 * Errors: W4A8_ERR_SCALE_RANGE if max S > 32767; W4A8_ERR_OVERFLOW_BOUND if
 * 127*127*group*colsum_max >= 2^31 (outputs are written in both cases).
 */
W4A8_API w4a8_status pack_w8_groupwise(const float* w, int64_t K, int64_t N, int32_t group, int32_t alpha_in,
                              int8_t* w8, float* s_g, int16_t* S, int32_t* alpha_out_host,
                              int64_t* colsum_max_host, void* workspace, void* stream);

/*
 * Bytes of workspace the GEMMs below need for (M, N, K, group) on the current
 * device (0 when they need none).  path: 0 integer scale, 1 float scale,
 * 2 the W8A8 integer-scale GEMM.
 * The workspace must be zero-filled before its first use.  Its first 4096
 * bytes hold arrival counters that every successful call leaves at zero
 * again (the rest is scratch), so one allocation of the largest size needed
 * serves any sequence of calls that run one after another; calls that
 * overlap on the GPU need one workspace each.  After an error or a timeout,
 * zero it again.
 */
W4A8_API int64_t w4a8_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int32_t group, int32_t path);

/*
 * W4A8 GEMM with integer group scales (the Integer-Scale scheme).
 * (Integer Scale summary §4 / Fig. 3(c); "Quantization" notes 矩阵乘法中的量化计算.)
 * Kernels by shape (256 <= K <= 16384 for the first): M <= 2, or M <= 4 with
 * at most 32 MB of packed weights, a CUDA-core kernel that streams the weights
 * (no workspace); otherwise the tcgen05 kernel with token tiles of 16..128.
 *   P_g[m,n] = sum_{k in g} q_x[m,k] q_w[k,n]            (int8 x int4 -> int32, tensor cores)
 *   acc[m,n] = sum_g S[g,n] * P_g[m,n]                    (int32, exact)
 *   y[m,n]   = fl_out(fl32(acc) * fl32(s_a[m] / alpha))   (one conversion per output)
 * q_x, s_a   device, [M, K] int8 and [M] float32 (from quantize_act_per_token)
 * w_packed   device, [N, K/2] uint8; S device [K/group, N] int16 (from pack_w4_groupwise)
 * alpha      power of two, 1 <= alpha <= 2^30
 * M >= 0 (0 is a no-op), N % 8 == 0, K % 128 == 0, group % 128 == 0, K % group == 0,
 *            and ceil(N/128) * ceil(M/BT) * (K/group) < 2^31 with BT the token tile
 *            (16, 32, 64 or 128, the smallest that holds M, capped at 128);
 *            otherwise W4A8_ERR_SHAPE
 * y          device, [M, N] of y_dtype: W4A8_F16, W4A8_F32, or W4A8_I32 (acc itself)
 * workspace  device, >= w4a8_gemm_workspace_size(M, N, K, group, 0) bytes (may be
 *            NULL when that size is 0), zero-filled, see above
 * Precondition (established by pack_w4_groupwise): the worst-case accumulator
 * 127*7*group*max_n sum_g |S[g,n]| stays below 2^31.
 * With 128-token tiles, a CTA whose scales S[g,n] all lie in [0, 16] (or
 * reach 17 or 18 only in groups without the code -8) writes S*q (then exact
 * in int8) as the MMA operand and sums the whole K in one accumulator: the
 * same acc, with no per-group multiply.
 */
W4A8_API w4a8_status w4a8_gemm_intscale(const int8_t* q_x, const float* s_a, const uint8_t* w_packed,
                               const int16_t* S, int32_t alpha, int64_t M, int64_t N, int64_t K,
                               int32_t group, void* y, int32_t y_dtype, void* workspace,
                               int64_t workspace_bytes, void* stream);

/*
 * The whole integer-scale linear layer from unquantized tokens: per-token
 * quantization, then the W4A8 integer-scale GEMM (Integer Scale summary,
 * Fig. 3(c): int8 tokens, int4 weights, integer group scales, one rescale).
 *   q_x, s_a = quantize_act_per_token(x);  y = w4a8_gemm_intscale(q_x, s_a, ...)
 * With one token and 256 <= K <= 16384 it is one kernel: every CTA quantizes
 * the token itself (the same codes and scale, bit for bit, as
 * quantize_act_per_token) and streams its weight columns on the CUDA cores.
 * With 2 to 4 tokens it is that kernel only when q_x / s_a are not given.
 * Otherwise it is the two calls above, chained on `stream`.  Every route
 * gives the same outputs bit for bit.
 * x, x_dtype, M, K, ldx   as quantize_act_per_token (W4A8_F32 or W4A8_BF16)
 * w_packed, S, alpha, N, group, y, y_dtype, workspace   as w4a8_gemm_intscale
 * q_x, s_a   device, [M, K] int8 and [M] float32: written with the token codes
 *            and scales when given (may be NULL when M <= 4 and
 *            256 <= K <= 16384); required otherwise (W4A8_ERR_INVALID_ARG),
 *            s_a then 16-byte aligned
 * Errors: as quantize_act_per_token and w4a8_gemm_intscale.
 */
W4A8_API w4a8_status w4a8_linear_intscale(const void* x, int32_t x_dtype, int64_t M, int64_t K, int64_t ldx,
                                         const uint8_t* w_packed, const int16_t* S, int32_t alpha, int64_t N,
                                         int32_t group, void* y, int32_t y_dtype, int8_t* q_x, float* s_a,
                                         void* workspace, int64_t workspace_bytes, void* stream);

/*
 * Weight-side zero-point term for asymmetric activations.
 * ("Quantization" notes, 矩阵乘法中的量化计算: with Z_W = 0 the integer part of
 *  the product is q_W q_X - Z_X q_W, and the weight-dependent correction can
 *  be precomputed; with integer group scales it is one int32 per column.)
 *   zc[n] = sum_g S[g,n] * sum_{k in g} q_w[k,n]    (two's-complement int32)
 * w_packed  device, [N, K/2] uint8, 16-byte aligned; S device [K/group, N] int16
 *           (from pack_w4_groupwise or pack_w4_groupwise_range)
 * K, N      K % group == 0, group % 32 == 0; otherwise W4A8_ERR_SHAPE
 * qmin      the code range the weights were packed with: -7 ([-7, 7]) or -8 ([-8, 7])
 * colsum_max  max_n sum_g |S[g,n]| as the pack call reported it (colsum_max_host)
 * zc        device, [N] int32, written
 * Errors: W4A8_ERR_OVERFLOW_BOUND, before anything is launched, when
 * 255 * |qmin| * group * colsum_max >= 2^31: the asymmetric GEMM's accumulator
 * would not be exact in int32 for every input (codes minus zero points span
 * 255 values); W4A8_ERR_INVALID_ARG for a NULL pointer, another qmin or a
 * negative colsum_max; W4A8_ERR_ALIGN unless w_packed is 16-byte, S 2-byte
 * and zc 4-byte aligned.
 */
W4A8_API w4a8_status w4_zero_point_term(const uint8_t* w_packed, const int16_t* S, int64_t K, int64_t N,
                                        int32_t group, int32_t qmin, int64_t colsum_max, int32_t* zc,
                                        void* stream);

/*
 * W4A8 integer-scale GEMM of asymmetric token codes (from
 * quantize_act_per_token_asym).  ("Quantization" notes, 矩阵乘法中的量化计算,
 *  with Z_W = 0 and Z_X = z_a[m]; Integer Scale summary §4.)
 *   acc[m,n] = sum_g S[g,n] * sum_{k in g} (q_x[m,k] - z_a[m]) q_w[k,n]
 *            = (the w4a8_gemm_intscale accumulator) - z_a[m] * zc[n]
 *   y[m,n]   = fl_out(fl32(acc) * fl32(s_a[m] / alpha))
 * The subtraction happens once per output, in the final pass (of the tile,
 * or of the decode kernel, which takes the same shapes as in
 * w4a8_gemm_intscale), in two's-complement int32 arithmetic: the
 * intermediate terms may wrap, the
 * result is exact when acc itself fits in int32, which holds when
 * 255*qw*group*max_n sum_g |S[g,n]| < 2^31 (255 = the widest |q_x - z_a|;
 * qw = 7, or 8 for codes in the full range [-8, 7]); w4_zero_point_term
 * refuses weights that break this bound, so a zc it wrote meets it.
 * z_a        device, [M] int32 (4-byte aligned)
 * zc         device, [N] int32 from w4_zero_point_term (4-byte aligned)
 * Other arguments, workspace (path 0), output (W4A8_I32: acc itself) and
 * errors as in w4a8_gemm_intscale.
 */
W4A8_API w4a8_status w4a8_gemm_intscale_asym(const int8_t* q_x, const float* s_a, const int32_t* z_a,
                                             const uint8_t* w_packed, const int16_t* S, const int32_t* zc,
                                             int32_t alpha, int64_t M, int64_t N, int64_t K, int32_t group,
                                             void* y, int32_t y_dtype, void* workspace, int64_t workspace_bytes,
                                             void* stream);

/*
 * W8A8 GEMM with integer group scales: the integer-scale GEMM above with
 * 8-bit weight codes w8 [N, K] int8 (from pack_w8_groupwise) instead of packed
 * int4.  acc[m,n] = sum_g S[g,n] * P_g[m,n] in int32 with
 * P_g[m,n] = sum_{k in g} q_x[m,k] * w8[n,k]; y = acc * s_a[m] / alpha.
 * Arguments, precondition (now 127*127*group*max_n sum_g |S[g,n]| < 2^31),
 * workspace (w4a8_gemm_workspace_size with path 2), output and errors as in
 * w4a8_gemm_intscale.  One or two tokens (three or four while w8 takes at
 * most 32 MB), 256 <= K <= 16384, run the CUDA-core decode kernel on the
 * 8-bit codes as stored, with no workspace; other shapes run the tiles.
 */
W4A8_API w4a8_status w8a8_gemm_intscale(const int8_t* q_x, const float* s_a, const int8_t* w8, const int16_t* S,
                               int32_t alpha, int64_t M, int64_t N, int64_t K, int32_t group, void* y,
                               int32_t y_dtype, void* workspace, int64_t workspace_bytes, void* stream);

/*
 * The integer-scale GEMM above with its workspace in a fixed device array of
 * the library instead of a caller buffer, so that a call allocates nothing.
 * The paper has no counterpart: it is a deployment convenience of this
 * library, the computation is w4a8_gemm_intscale's.
 * Arguments as w4a8_gemm_intscale without workspace and workspace_bytes.
 * Limit: calls whose w4a8_gemm_workspace_size(M, N, K, group, 0) exceeds
 * W4A8_STATIC_WORKSPACE_BYTES (8 MiB: every plan with token tiles up to 64,
 * i.e. M <= 64, and any plan that splits no tile) are refused with
 * W4A8_ERR_WORKSPACE before anything is launched.
 * The array is one per device and shared by every call of this entry point
 * on that device: calls whose kernels overlap on the GPU (different streams
 * without ordering) race on it and must not be issued.  Its first 4096 bytes
 * are arrival counters that start at zero (at library load) and that every
 * completed call leaves at zero; the rest needs no clearing.
 * The first call on a device looks the array's address up (a CUDA runtime
 * call that must not run inside a stream capture), so make one call on each
 * device before capturing any.
 */
#define W4A8_STATIC_WORKSPACE_BYTES (8 << 20)
W4A8_API w4a8_status w4a8_gemm_intscale_static_ws(const int8_t* q_x, const float* s_a, const uint8_t* w_packed,
                                                 const int16_t* S, int32_t alpha, int64_t M, int64_t N, int64_t K,
                                                 int32_t group, void* y, int32_t y_dtype, void* stream);

/*
 * Mixture-of-experts layer in one grouped call: the integer-scale W4A8 GEMM of
 * every expert over the token rows routed to it.  (Integer Scale summary
 * §5.3: the method applied to Mixtral 8x7B; every expert's linear layer is a
 * fine-grained W4A8 GEMM and the amplifier is one per layer, shared by all
 * experts.)
 *   for every routed row i of expert e (offsets[e] <= i < offsets[e+1]):
 *     y[out_row ? out_row[i] : i, :] = the w4a8_gemm_intscale row of token
 *         row_index[i] with expert e's w_packed[e], S[e] and the shared alpha
 * Everything the routing decides is read on the device, so a router kernel
 * earlier in the stream can produce it without a host round trip: a small
 * setup kernel turns the offsets into the schedule and each expert's weight
 * tensor map (in the workspace), then one persistent launch of the
 * w4a8_gemm_intscale tiles covers every (expert, tile, group) step.  Token
 * rows are gathered from q_x by index, four rows per copy (no gathered copy
 * is made), or, with row_index NULL, q_x holds the routed rows themselves
 * (quantize_act_routed) and each tile's rows are read as one block (measured
 * about half the time on a Mixtral-shaped layer: the four-row copies bound
 * the gathered form).
 * q_x, s_a   device, [T, K] int8 and [T] float32: every token quantized once
 *            (quantize_act_per_token), or, with row_index NULL, the routed rows
 *            (T >= R; quantize_act_routed); q_x 16-byte, s_a 4-byte aligned
 * row_index  device, [R] int32 or NULL: the token of each routed row, rows
 *            grouped by expert (expert 0 first).  A token outside [0, T) gives
 *            that row zero output and sets W4A8_ERR_INVALID_ARG in the device
 *            status word.  NULL: routed row i is row i of q_x
 * expert_offsets  device, [E+1] int64 (8-byte aligned): offsets[0] = 0,
 *            non-decreasing, offsets[E] = R; anything else makes the call
 *            write nothing and set W4A8_ERR_INVALID_ARG in the device status
 * out_row    device, [R] int32 or NULL: the output row of each routed row, e.g.
 *            token * top_k + slot to return rows in (token, slot) order; NULL
 *            writes routed row i to row i.  A row outside [0, y_rows) is not
 *            written and sets W4A8_ERR_INVALID_ARG in the device status word
 * w_packed, S  device arrays (8-byte aligned) of E device pointers: expert e's
 *            packed weights [N, K/2] (16-byte aligned) and integer scales
 *            [K/group, N] (2-byte aligned), all packed with the same alpha (pack
 *            each expert's s_g with S = NULL, run w4a8_amplifier_search over all
 *            of them, pack every expert with it).  Experts with no rows may
 *            have NULL pointers; a NULL or misaligned pointer of an expert with
 *            rows makes the call write nothing and set W4A8_ERR_INVALID_ARG
 * E          1 <= E <= 256; R the routed rows (T * top_k), 0 <= R < 2^31;
 *            N, K, group as for w4a8_gemm_intscale
 * y          device, [y_rows, N] of y_dtype (W4A8_F16, W4A8_F32, W4A8_I32),
 *            16-byte aligned; y_rows >= R when out_row is NULL
 * workspace  device, >= w4a8_grouped_workspace_size(E, N, K, group) bytes,
 *            16-byte aligned, zero-filled before its first use; its first 4096
 *            bytes are counters that every completed call leaves at zero, the
 *            rest holds partial sums, the tensor maps and the schedule
 * Asynchronous on `stream`: two launches (setup, then the GEMM), chained with
 * programmatic dependent launch.
 */
W4A8_API int64_t w4a8_grouped_workspace_size(int32_t E, int64_t N, int64_t K, int32_t group);
W4A8_API w4a8_status w4a8_gemm_intscale_grouped(const int8_t* q_x, const float* s_a, int64_t T,
                                               const int32_t* row_index, const int64_t* expert_offsets,
                                               const int32_t* out_row, const uint8_t* const* w_packed,
                                               const int16_t* const* S, int32_t alpha, int32_t E, int64_t R,
                                               int64_t N, int64_t K, int32_t group, void* y, int32_t y_dtype,
                                               int64_t y_rows, void* workspace, int64_t workspace_bytes,
                                               void* stream);

/*
 * W4A8 GEMM with float group scales, the comparison path.
 * (Integer Scale summary §3.2 / Fig. 3(b): every group's int32 result is
 *  converted to fp32 and multiplied by its float scale.)
 *   y[m,n] = fl_out(s_a[m] * sum_g s_g[g,n] * float(P_g[m,n]))   (fp32, group order)
 * Arguments as w4a8_gemm_intscale with float s_g [K/group, N] in place of S and
 * alpha; y_dtype W4A8_F16 or W4A8_F32; workspace size from path 1.
 */
W4A8_API w4a8_status w4a8_gemm_floatscale(const int8_t* q_x, const float* s_a, const uint8_t* w_packed,
                                 const float* s_g, int64_t M, int64_t N, int64_t K, int32_t group,
                                 void* y, int32_t y_dtype, void* workspace, int64_t workspace_bytes,
                                 void* stream);

/*
 * Measurement aid, not a step of the method: the int8 tensor-core rate of this
 * GPU.  Launches one CTA per SM; each issues iters x 4 back-to-back
 * tcgen05.mma.kind::i8 of shape 128 x n x 32 (signed int8, int32 accumulator
 * in TMEM) on operands already on chip: the weight-side operand from shared
 * memory (a_in_tmem = 0) or from TMEM (a_in_tmem != 0, as the W4A8 GEMM feeds
 * its unpacked weights), the token-side operand from shared memory.  No loads
 * from global memory and no epilogue.  Asynchronous on `stream`: time it with
 * events around the call.
 * iters      1 .. 2^30; n: 16 .. 256, a multiple of 16; otherwise W4A8_ERR_SHAPE
 * grid_host  host, written: the CTAs launched (the SM count)
 * ops_host   host, written: int8 operations of the launch, 2*128*n*128*iters*grid
 * A wait that runs out sets W4A8_ERR_TIMEOUT in the device status word.
 */
W4A8_API w4a8_status w4a8_tensor_i8_peak_probe(int64_t iters, int32_t n, int32_t a_in_tmem, int32_t* grid_host,
                                              double* ops_host, void* stream);

/*
 * How long the GEMMs' waits inside a kernel may last: the pipeline waits
 * between the roles of a CTA and a split tile's wait for the other CTAs'
 * partial sums, in SM clock cycles (default 2^31, about one second).  A wait
 * that runs out makes the kernel leave early (after the copies and MMAs it has
 * in flight complete) with W4A8_ERR_TIMEOUT in the device status word; the
 * call's output is then undefined and its workspace must be zeroed again.
 * cycles <= 0 restores the default.  Applies to launches made after the call,
 * process-wide.  Returns the previous limit.  A diagnostic and test aid: a
 * short limit turns a stall (another kernel holding SMs, for instance) into an
 * error the host can read.
 */
W4A8_API int64_t w4a8_set_wait_limit(int64_t cycles);

/*
 * The CUDA runtime error code (cudaError_t) behind the last W4A8_ERR_CUDA that
 * a call of this library returned on the calling thread (0 if none); with
 * clear != 0 the record is reset.  w4a8_cuda_error_string names a code.
 */
W4A8_API int32_t w4a8_last_cuda_error(int32_t clear);
W4A8_API const char* w4a8_cuda_error_string(int32_t code);

/*
 * Reads (and with clear != 0 resets) the device status word of the current
 * device: 0, or the last device-side error: W4A8_ERR_TIMEOUT (a bounded wait
 * ran out) or W4A8_ERR_INVALID_ARG (bad routing data in
 * w4a8_gemm_intscale_grouped).  Synchronous.  The word keeps only the last error,
 * so clearing any nonzero status also zeroes the arrival counters of the
 * library's own workspace (w4a8_static_workspace_reset); caller workspaces
 * must be zeroed by the caller.
 */
W4A8_API w4a8_status w4a8_device_status(int32_t* code_host, int32_t clear);

/*
 * Zeroes the split-tile arrival counters of the library's own workspace (the
 * one w4a8_gemm_intscale_static_ws uses) on the current device, if that
 * workspace has been set up there; synchronous.  Needed after a call that
 * failed or timed out, which may leave counts behind.  Allocates nothing.
 */
W4A8_API w4a8_status w4a8_static_workspace_reset(void);

#ifdef __cplusplus
}
#endif

#endif /* W4A8_INTSCALE_H */
