/*
 * bitlinear.h -- C ABI of libbitlinear.so, the B200 (sm_100a) BitLinear
 * W1.58A8 forward: ternary weights {-1, 0, +1} with one scale per matrix,
 * int8 activations quantised per token by absmax, int32 accumulation and a
 * fused rescale.
 *
 * Sources (web pages):
 *   [MMF] DataCamp blog "MatMul-free language models" (Dutch): section
 *         "MatMul vervangen door ternaire bewerkingen" (absmean ternarisation;
 *         a multiply by -1/0/+1 is a negate/zero/pass-through), figure item
 *         "RMS norm" (normalise activations before quantisation), section
 *         "Kerncomponenten: MLGRU en GLU" (the MatMul-free GLU).
 *   [BNC] unite.ai "Microsofts Inference Framework bringt 1-Bit grosse
 *         Sprachmodelle auf lokale Geraete" (German): section "Ternaeres
 *         Gewichtssystem" (1.58-bit ternary weights), section "Mathematische
 *         Grundlagen" eq. 2 "Aktivierungsquantisierung" and eq. 3
 *         "BitLinear-Betrieb", section "Implementierungshinweise" (the
 *         quantise -> ternary matmul -> scale shape of a forward call); the
 *         1-bit weights of the same section, item 1 "Gewichtsbinarisierung";
 *         section "Gruppenquantisierung und -normalisierung" (group quantisation).
 *
 * Conventions for every call:
 *   - Every pointer argument is a DEVICE pointer owned by the caller (the
 *     library allocates nothing and frees nothing), 16-byte aligned.  Outputs
 *     must not overlap inputs.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls only enqueue work on it and never synchronise, except
 *     bitlinear_device_status(), which says so.
 *   - Shapes: M tokens, K input features, N output features.  x is [M, K]
 *     row-major, W is [N, K] row-major (nn.Linear out x in), y is [M, N]
 *     row-major.  Sizes are int64_t and must be >= 1.
 *   - Arguments are validated on the host before any launch; on error nothing
 *     is launched and a nonzero bl_status is returned.  Device faults are not
 *     used for error reporting.  Non-finite inputs (NaN, Inf) give
 *     unspecified results.
 *   - A nonzero return after a launch (BL_ERR_CUDA) carries the CUDA error of
 *     the launch; the stream is otherwise left as it was.
 */
#ifndef BITLINEAR_H
#define BITLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int bl_status;

enum {
    BL_OK = 0,
    BL_ERR_NULL = 1,       /* a required pointer is NULL */
    BL_ERR_SHAPE = 2,      /* a size is < 1, too large, or violates a divisibility rule */
    BL_ERR_ALIGN = 3,      /* a pointer is not 16-byte aligned */
    BL_ERR_DTYPE = 4,      /* unknown dtype or combine enum */
    BL_ERR_WORKSPACE = 5,  /* workspace NULL or smaller than the *_workspace() size */
    BL_ERR_DEVICE = 6,     /* no CUDA device, or current device is not compute capability 10.x */
    BL_ERR_CUDA = 7,       /* a launch or runtime call failed */
    BL_ERR_TIMEOUT = 8,    /* a bounded on-device wait expired (reported by bitlinear_device_status) */
    BL_ERR_ALIAS = 9       /* an output overlaps an input */
};

enum { BL_F32 = 0, BL_BF16 = 1, BL_I8 = 2 /* already-quantised x_q with per-token gamma */ };

/* Largest K accepted (keeps every int32 partial of the contraction exact). */
#define BL_MAX_K 262144

/* Human-readable name of a status code (static string, never NULL). */
const char* bitlinear_status_string(bl_status s);

/* ------------------------------------------------------------------------ */
/* Offline weight preparation                                                */
/* ------------------------------------------------------------------------ */

/* Bytes of device workspace bitlinear_quantize_weights needs (any N, K). */
size_t bitlinear_quantize_weights_workspace(int64_t N, int64_t K);

/*
 * absmean ternarisation, [MMF] "MatMul vervangen door ternaire bewerkingen":
 *   beta   = mean over all N*K elements of |W|          (one scale per matrix)
 *   W_t    = clip(round(W / (beta + eps)), -1, 1)        (ties to even)
 * beta is the exact sum of |W| rounded once to binary64, divided by N*K in
 * binary64 and rounded to binary32, for every finite W (subnormals
 * included).  The sum is taken in exact integer arithmetic, so it does not
 * depend on thread order: an element within 2^38 of max|W| is an integer on
 * the grid 2^(E-188) (E the biased exponent of max|W|), a smaller one an
 * integer on the grid 2^-149, and all are added without rounding before the
 * one conversion.  The divisor beta + eps and the quotient are binary32
 * (IEEE add, IEEE divide).
 *   W    [N, K] float32, device, read only
 *   W_t  [N, K] int8 out, values in {-1, 0, 1}
 *   beta [1] float32 out (stays on the device)
 *   ws   >= bitlinear_quantize_weights_workspace(N, K) bytes of device scratch
 *        (contents on entry do not matter; calls sharing a ws must not overlap)
 * eps must be finite and >= 0 (1e-5 in the workloads); an all-zero W gives
 * beta = 0 and W_t = 0.
 */
bl_status bitlinear_quantize_weights(const float* W, int64_t N, int64_t K, float eps,
                                     int8_t* W_t, float* beta, void* ws, size_t ws_bytes,
                                     void* stream);

/*
 * 2-bit packing of ternary weights ([BNC] "Ternaeres Gewichtssystem": three
 * states per weight, stored here in 2 bits, 16 per uint32).  Code c = w + 1
 * in {0, 1, 2}.  For row n and word j, the trit at k = 16j + 4s + b
 * (s, b in 0..3) sits at bits [8b + 2s, 8b + 2s + 1] of W_p[n, j], so that
 * (word >> 2s) & 0x03030303 holds the codes of k = 16j+4s .. 16j+4s+3 in
 * its four bytes.  An all-zero group of 16 trits packs to 0x55555555.
 *   W_t [N, K] int8 in, values must be in {-1, 0, 1} (others: unspecified)
 *   W_p [N, K/16] uint32 out
 * K % 16 == 0.
 */
bl_status bitlinear_pack(const int8_t* W_t, int64_t N, int64_t K, uint32_t* W_p, void* stream);

/* ------------------------------------------------------------------------ */
/* Per-token forward                                                         */
/* ------------------------------------------------------------------------ */

/*
 * Per-token absmax int8 activation quantiser, [BNC] eq. 2
 * "Aktivierungsquantisierung" with Q_b = 127 and a symmetric clamp:
 *   gamma_m = max(max_k |x[m, k]|, 1e-5)                  (binary32)
 *   s_m     = 127 / gamma_m                               (binary32 IEEE divide)
 *   x_q     = clip(rint(x[m, k] * s_m), -127, 127)        (binary32 multiply, ties to even)
 *   x     [M, K] float32 (x_dtype BL_F32) or bfloat16 (BL_BF16), in
 *   x_q   [M, K] int8 out
 *   gamma [M] float32 out
 * K % 16 == 0, K <= BL_MAX_K.
 */
bl_status bitlinear_quant_act(const void* x, int x_dtype, int64_t M, int64_t K,
                              int8_t* x_q, float* gamma, void* stream);

/* Bytes of device workspace bitlinear_forward needs for this shape (may be 0). */
size_t bitlinear_forward_workspace(int64_t M, int64_t N, int64_t K);

/*
 * BitLinear forward on quantised inputs, [BNC] eq. 3 "BitLinear-Betrieb",
 * with the multiplies of [MMF] replaced by add / subtract / skip:
 *   acc[m, n] = sum_k W_t[n, k] * x_q[m, k]               (int32, exact)
 *   y[m, n]   = (float)acc[m, n] * ((beta * gamma_m) / 127)  (binary32, this order)
 * and for y_dtype BL_BF16 the binary32 value rounded to nearest-even bf16.
 *   x_q   [M, K] int8, gamma [M] float32, W_p [N, K/16] uint32 (bitlinear_pack
 *         layout), beta [1] float32 -- all inputs
 *   y     [M, N] float32 or bfloat16 out
 *   ws    >= bitlinear_forward_workspace(M, N, K) bytes (may be NULL when that is 0)
 * K % 64 == 0, K <= BL_MAX_K.  By default M <= 4 runs the decode GEMV on
 * CUDA cores, 5 <= M <= 16 a decode kernel on the tcgen05 int8 tensor cores
 * (where x_hat fits its shared memory; above 8 tokens only while each CTA's
 * rows fit one 128-lane tile) and larger M the GEMM on the tensor cores
 * (bitlinear_set_decode_engine selects other kernels for M <= 64;
 * bitlinear_forward_path reports the choice).  All give identical results.
 *
 * The forward kernels begin streaming W_p and read beta before the kernel
 * queued ahead of them on the stream has finished (programmatic dependent
 * launch); x_q and gamma are read only after it finished.  W_p and beta must
 * therefore not be written by a kernel that is still running when the
 * forward is launched: kernels without programmatic dependent launch, this
 * library's own included, always finish first.
 */
bl_status bitlinear_forward(const int8_t* x_q, const float* gamma, int64_t M, int64_t K,
                            const uint32_t* W_p, const float* beta, int64_t N,
                            void* y, int y_dtype, void* ws, size_t ws_bytes, void* stream);

/* Bytes of device workspace bitlinear_forward_fp needs for this shape (may be 0). */
size_t bitlinear_forward_fp_workspace(int64_t M, int64_t N, int64_t K);

/*
 * Quantise + forward in one call, the shape of the forward function sketched
 * in [BNC] "Implementierungshinweise" (quantise the input, ternary matmul,
 * scale): bitlinear_quant_act(x) followed by bitlinear_forward, with results
 * bit-identical to those two calls.  For M <= 4 tokens with
 * (M rounded up to 1, 2 or 4) * K <= 65536 the quantiser runs in the GEMV
 * prologue (one kernel, workspace 0); otherwise x_q and gamma are staged in
 * the workspace and the two kernels run back to back.
 *   x  [M, K] float32 (BL_F32) or bfloat16 (BL_BF16) in; other arguments as
 *   for bitlinear_forward.  K % 64 == 0, K <= BL_MAX_K.
 */
bl_status bitlinear_forward_fp(const void* x, int x_dtype, int64_t M, int64_t K, const uint32_t* W_p,
                               const float* beta, int64_t N, void* y, int y_dtype, void* ws, size_t ws_bytes,
                               void* stream);

/* One problem of a bitlinear_forward_fp_batch call. */
typedef struct {
    const void* x;          /* [M, K] activations (x_dtype of the call), in */
    const float* gamma;     /* [M] per-token scale when x_dtype is BL_I8 (x is x_q), else unused */
    const uint32_t* W_p;    /* [N, K/16] packed weights (bitlinear_pack layout), in */
    const float* beta;      /* [1] absmean scale of W_p, in */
    void* y;                /* [M, N] output (y_dtype of the call), out */
    int64_t K, N;
} bl_problem;

/* Most problems one bitlinear_forward_fp_batch call takes. */
#define BL_BATCH_MAX 8

/*
 * Several independent decode projections in one launch: bitlinear_forward_fp
 * on each problem (same results, bit for bit), or bitlinear_forward when
 * x_dtype is BL_I8 (x holds x_q and gamma the per-token scales), e.g. the q / k / v
 * projections of one token, gate and up, or projections of different layers
 * whose inputs are ready.  The problems share M (<= 4), x_dtype and y_dtype;
 * each needs (M rounded up to 1, 2 or 4) * K <= 65536, K % 64 == 0.  Every SM
 * runs one CTA per problem, so their HBM streams and fixed latencies overlap.
 * Outputs must not overlap any input or each other.
 *   problems: host array of `count` descriptors (1 <= count <= BL_BATCH_MAX),
 *             read during the call only.
 */
bl_status bitlinear_forward_fp_batch(const bl_problem* problems, int count, int64_t M, int x_dtype, int y_dtype,
                                     void* stream);

/*
 * Inspection variant of bitlinear_forward: writes the int32 accumulators
 * acc[M, N] = sum_k W_t[n, k] * x_q[m, k] instead of y (same kernels, same
 * dispatch, rescale skipped).  For exact comparisons in tests.
 */
bl_status bitlinear_forward_acc(const int8_t* x_q, int64_t M, int64_t K,
                                const uint32_t* W_p, int64_t N, int32_t* acc,
                                void* ws, size_t ws_bytes, void* stream);

/* Rows the built-in scratch of bitlinear_forward_noalloc holds (64 KiB of int32). */
#define BL_NOALLOC_MAX_M 16384

/*
 * bitlinear_forward for callers that cannot allocate device memory -- a C
 * runtime with a fixed arena and no device allocator to hand the library,
 * or code being recorded into a stream capture where an allocation is not
 * allowed.  The pages have no counterpart: this is a library convenience.
 * Same arguments, kernels, dispatch and results as bitlinear_forward, without
 * ws/ws_bytes: the M int32 row sums the GEMM path (M > 4) needs live in a
 * static device array of the library (BL_NOALLOC_MAX_M entries, held by every
 * device that loads the library until exit); the CUDA-core and swap-AB
 * decode kernels need no scratch.
 *   - M > BL_NOALLOC_MAX_M returns BL_ERR_WORKSPACE (scratch too small), with
 *     nothing launched.
 *   - The first call on a device looks up the array's device address and
 *     checks the device (no allocation); make that first call before any
 *     stream capture on that device.
 *   - Every call on a device shares the array and overwrites the rows it
 *     uses before reading them; calls that overlap on the GPU (for example on
 *     two streams) race on it and must be serialised by the caller.
 *   - No cudaMalloc, cudaFree or allocating library routine is called.
 */
bl_status bitlinear_forward_noalloc(const int8_t* x_q, const float* gamma, int64_t M, int64_t K,
                                    const uint32_t* W_p, const float* beta, int64_t N,
                                    void* y, int y_dtype, void* stream);

/* ------------------------------------------------------------------------ */
/* 1-bit weight variant                                                      */
/* ------------------------------------------------------------------------ */

/*
 * [BNC] "Mathematische Grundlagen", item 1 "Gewichtsbinarisierung", eq. 1:
 * the weights are centred on their mean and binarised,
 *   W_b = Sign(W - alpha),  alpha = mean(W),  Sign(d) = +1 for d > 0, else -1
 * (so an element equal to alpha gets -1), and eq. 3 applies unchanged with
 * W_f = W_b.  The forward below is the same contraction as for ternary
 * weights, restricted to w in {-1, +1} and stored in 1 bit per weight.
 */

/* Bytes of device workspace bitlinear_binarize_weights needs (any N, K). */
size_t bitlinear_binarize_weights_workspace(int64_t N, int64_t K);

/*
 * Binarisation of a full-precision matrix, eq. 1 above.
 *   alpha = (float)(S / (N*K))   S = the exact sum of W rounded once to
 *                                binary64, divided in binary64
 *   beta  = mean |W| exactly as bitlinear_quantize_weights computes it (the
 *           page names beta a scaling factor without a formula; this library
 *           reads it as the absmean scale of the ternary weights)
 *   W_b   = +1 where (W - alpha) > 0 in binary32, else -1
 *   W     [N, K] float32 in
 *   W_b   [N, K] int8 out, values in {-1, +1}
 *   alpha [1] float32 out, beta [1] float32 out (distinct buffers)
 *   ws    >= bitlinear_binarize_weights_workspace(N, K) bytes of device scratch
 * K % 32 == 0.  The sums of the positive and of the negative elements are
 * exact integers (as for bitlinear_quantize_weights) and do not depend on
 * thread order, so alpha and beta are the exact means defined above for
 * every finite W.
 */
bl_status bitlinear_binarize_weights(const float* W, int64_t N, int64_t K, int8_t* W_b, float* alpha,
                                     float* beta, void* ws, size_t ws_bytes, void* stream);

/*
 * 1-bit packing, 32 weights per uint32.  For row n and word j, the weight at
 * k = 32j + 4s + b (s in 0..7, b in 0..3) is bit 8b + s of W_p[n, j]: set for
 * w > 0 (+1), clear otherwise (-1), so that (word >> s) & 0x01010101 holds
 * the signs of k = 32j+4s .. 32j+4s+3 in its four bytes.
 *   W_b [N, K] int8 in (values <= 0 are stored as -1)
 *   W_p [N, K/32] uint32 out
 * K % 32 == 0.
 */
bl_status bitlinear_pack_bits(const int8_t* W_b, int64_t N, int64_t K, uint32_t* W_p, void* stream);

/* Bytes of device workspace bitlinear_forward_binary needs for this shape (may be 0). */
size_t bitlinear_forward_binary_workspace(int64_t M, int64_t N, int64_t K);

/*
 * BitLinear forward with 1-bit weights, eq. 3 with W_f = W_b:
 *   acc[m, n] = sum_k W_b[n, k] * x_q[m, k]
 *             = 2 * sum_{k: W_b = +1} x_q[m, k] - sum_k x_q[m, k]  (int32, exact)
 *   y[m, n]   = (float)acc[m, n] * ((beta * gamma_m) / 127)      (binary32, this order)
 * Arguments as for bitlinear_forward, with W_p [N, K/32] in the
 * bitlinear_pack_bits layout.  K % 128 == 0, K <= BL_MAX_K.  M <= 4 tokens
 * (with M rounded up to 1, 2 or 4, times K <= 65536) run the CUDA-core GEMV,
 * which streams 1 bit per weight; other shapes run the tcgen05 GEMM.  The
 * decode engine setting does not apply.  The same rule on W_p and beta as
 * for bitlinear_forward (they are read before the preceding kernel ends).
 */
bl_status bitlinear_forward_binary(const int8_t* x_q, const float* gamma, int64_t M, int64_t K,
                                   const uint32_t* W_p, const float* beta, int64_t N,
                                   void* y, int y_dtype, void* ws, size_t ws_bytes, void* stream);

/* Integer accumulators of bitlinear_forward_binary (same kernels, rescale skipped). */
bl_status bitlinear_forward_binary_acc(const int8_t* x_q, int64_t M, int64_t K,
                                       const uint32_t* W_p, int64_t N, int32_t* acc,
                                       void* ws, size_t ws_bytes, void* stream);

/* Bytes of device workspace bitlinear_forward_binary_fp needs for this shape (may be 0). */
size_t bitlinear_forward_binary_fp_workspace(int64_t M, int64_t N, int64_t K);

/*
 * bitlinear_quant_act(x) followed by bitlinear_forward_binary, bit-identical
 * to the two calls.  Where the GEMV runs (see above) the quantiser is fused
 * into its prologue and the workspace is 0.
 *   x [M, K] float32 (BL_F32) or bfloat16 (BL_BF16) in; other arguments as
 *   for bitlinear_forward_binary.  K % 128 == 0, K <= BL_MAX_K.
 */
bl_status bitlinear_forward_binary_fp(const void* x, int x_dtype, int64_t M, int64_t K, const uint32_t* W_p,
                                      const float* beta, int64_t N, void* y, int y_dtype, void* ws,
                                      size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* Decoder-block glue                                                        */
/* ------------------------------------------------------------------------ */

enum { BL_COMBINE_NONE = 0, BL_COMBINE_ADD = 1, BL_COMBINE_SILU_MUL = 2 };

/*
 * Fused combine + RMSNorm + int8 quantiser for the decoder block, one token
 * per row.  [MMF] figure item "RMS norm": activations are RMS-normalised
 * (gain 1) before quantisation; [MMF] "Kerncomponenten: MLGRU en GLU": the
 * GLU gates one BitLinear output with SiLU of the other.
 *   h[m, k] = a                                  (BL_COMBINE_NONE)
 *           = a + b            (binary32 add)     (BL_COMBINE_ADD)
 *           = (float)(silu(a) * b), silu(a) = a / (1 + exp(-a)), in binary64
 *                                                 (BL_COMBINE_SILU_MUL)
 *   rho_m   = (float)(1 / sqrt(mean_k h^2 + 1e-6))    (binary64, then rounded; the
 *             binary64 sum of squares is added in an order of the kernel's choosing,
 *             so rho can differ by one binary32 ulp from a sequential sum when that
 *             sum lies within its rounding error of a binary32 rounding boundary)
 * absmax quantisation is invariant under the positive per-token scale rho,
 * so the codes are those of bitlinear_quant_act applied to h, and
 *   gamma[m] = rho_m * max(max_k |h[m, k]|, 1e-5)       (binary32 multiply).
 *   a, b  [M, K] float32 in (b unused and may be NULL for BL_COMBINE_NONE)
 *   h     [M, K] float32 out, may be NULL (not written)
 *   x_q   [M, K] int8 out, may be NULL together with gamma (then only h is
 *         produced and no norm is computed)
 *   gamma [M] float32 out
 * K % 16 == 0, K <= BL_MAX_K.
 */
bl_status bitlinear_quant_act_rms(const float* a, const float* b, int combine, int64_t M, int64_t K,
                                  float* h, int8_t* x_q, float* gamma, void* stream);

/* ------------------------------------------------------------------------ */
/* Group quantisation                                                        */
/* ------------------------------------------------------------------------ */

/*
 * [BNC] section "Gruppenquantisierung und -normalisierung": weights and
 * activations are divided into G groups, each with its own parameters, so
 * that the groups can be processed in parallel without exchanging them.
 * Here the groups are G contiguous, equal blocks of the contraction
 * dimension: K_g = [g*K/G, (g+1)*K/G).  Group g of W (all rows, columns K_g)
 * has its absmean beta_g; group g of a token x_m has its absmax gamma_{m,g}.
 *   acc_g[m, n] = sum_{k in K_g} W_t[n, k] * x_q[m, k]                   (int32)
 *   y[m, n]     = sum over g = 0, 1, ... of (float)acc_g[m, n] * ((beta_g * gamma_{m,g}) / 127)
 * with every product, quotient and add one binary32 operation, the adds in
 * increasing g.  G = 1 is exactly the ungrouped path.
 *
 * Layouts are group-major, so every group is an ordinary matrix:
 *   W_t [G][N][K/G] int8; W_p [G][N][K/(16G)] uint32 = bitlinear_pack of W_t
 *       viewed as G*N rows of K/G trits; beta [G] float32;
 *   x_q [G][M][K/G] int8; gamma [M][G] float32.
 * 1 <= G <= BL_MAX_GROUPS, K % (64 G) == 0 for every call below.
 */
#define BL_MAX_GROUPS 8

/* Bytes of device workspace bitlinear_quantize_weights_grouped needs (4*N*K + a few KiB). */
size_t bitlinear_quantize_weights_grouped_workspace(int64_t N, int64_t K, int64_t G);

/*
 * Per-group absmean ternarisation: beta_g and W_t[:, K_g] exactly as
 * bitlinear_quantize_weights computes them for the matrix W[:, K_g] alone.
 *   W [N, K] float32 in; W_t [G][N][K/G] int8 out; beta [G] float32 out.
 * The workspace holds W regrouped to [G][N][K/G] (4*N*K bytes) and the sums.
 */
bl_status bitlinear_quantize_weights_grouped(const float* W, int64_t N, int64_t K, int64_t G, float eps,
                                             int8_t* W_t, float* beta, void* ws, size_t ws_bytes, void* stream);

/*
 * Per-token, per-group absmax quantiser: gamma[m][g] and the codes of
 * x[m, K_g] exactly as bitlinear_quant_act computes them for that block alone.
 *   x [M, K] float32 (BL_F32) or bfloat16 (BL_BF16) in;
 *   x_q [G][M][K/G] int8 out; gamma [M][G] float32 out.
 */
bl_status bitlinear_quant_act_grouped(const void* x, int x_dtype, int64_t M, int64_t K, int64_t G,
                                      int8_t* x_q, float* gamma, void* stream);

/* Bytes of device workspace bitlinear_forward_grouped and _grouped_acc need (> 0). */
size_t bitlinear_forward_grouped_workspace(int64_t M, int64_t N, int64_t K, int64_t G);

/*
 * Group-quantised forward (formula above).  The G contractions run as the
 * ungrouped ones would on each group (for M <= 4 tokens, with M rounded up to
 * 1, 2 or 4 times K/G <= 65536, all groups in one launch), writing int32
 * accumulators to the workspace; one more kernel applies the per-group scales
 * in order.  Arguments as for bitlinear_forward with the grouped layouts.
 */
bl_status bitlinear_forward_grouped(const int8_t* x_q, const float* gamma, int64_t M, int64_t K, int64_t G,
                                    const uint32_t* W_p, const float* beta, int64_t N, void* y, int y_dtype,
                                    void* ws, size_t ws_bytes, void* stream);

/*
 * The per-group accumulators of bitlinear_forward_grouped: acc_g[m, n] at
 * acc[g * S + m * N + n], S = M*N rounded up to a multiple of 4 (so acc holds
 * G*S int32).  For exact comparisons in tests.
 */
bl_status bitlinear_forward_grouped_acc(const int8_t* x_q, int64_t M, int64_t K, int64_t G, const uint32_t* W_p,
                                        int64_t N, int32_t* acc, void* ws, size_t ws_bytes, void* stream);

/* Bytes of device workspace bitlinear_forward_grouped_fp needs. */
size_t bitlinear_forward_grouped_fp_workspace(int64_t M, int64_t N, int64_t K, int64_t G);

/*
 * bitlinear_quant_act_grouped(x) then bitlinear_forward_grouped, bit-identical
 * to the two calls.  For one token (M = 1, K/G <= 65536) each group's slice of
 * x is contiguous: the quantiser then runs inside one GEMV launch over all
 * groups, which writes every group's binary32 term, and one more kernel adds
 * them in increasing g (2 launches).
 */
bl_status bitlinear_forward_grouped_fp(const void* x, int x_dtype, int64_t M, int64_t K, int64_t G,
                                       const uint32_t* W_p, const float* beta, int64_t N, void* y, int y_dtype,
                                       void* ws, size_t ws_bytes, void* stream);

/* Bytes of device workspace bitlinear_glu_forward needs for this shape. */
size_t bitlinear_glu_workspace(int64_t M, int64_t D, int64_t F);

/*
 * The MatMul-free GLU channel mixer, [MMF] "Kerncomponenten: MLGRU en GLU":
 * the input goes through two BitLinear layers, SiLU of one output is
 * multiplied elementwise by the other, and the gated result goes through a
 * third BitLinear.  Every BitLinear input is RMS-normalised before
 * quantisation ([MMF] figure item "RMS norm"), as bitlinear_quant_act_rms
 * does it, token by token:
 *   (x_q, gamma)   = quant_act_rms(x)                   codes shared by gate and up
 *   gate, up       = forward(x_q, gamma, W_gate | W_up)  [M, F] float32
 *   u              = SiLU(gate) * up                    (binary64, rounded once)
 *   (u_q, gamma_u) = quant_act_rms(u)
 *   y              = forward(u_q, gamma_u, W_down)       [M, D] float32
 * Results are bit-identical to those calls made one by one.  For M <= 4
 * tokens (with M rounded up to 1, 2 or 4, times D <= 65536) gate and up run
 * in one launch; otherwise each runs on the kernel bitlinear_forward picks.
 *   x       [M, D] float32 in
 *   W_gate, W_up [F, D/16] uint32 (bitlinear_pack layout), beta_gate, beta_up [1] float32, in
 *   W_down  [D, F/16] uint32, beta_down [1] float32, in
 *   y       [M, D] float32 out
 *   u       [M, F] float32 out, may be NULL (not written)
 *   ws      >= bitlinear_glu_workspace(M, D, F) bytes (holds x_q, gate, up, u_q, scales)
 * D % 64 == 0, F % 64 == 0, D and F <= BL_MAX_K.
 */
bl_status bitlinear_glu_forward(const float* x, int64_t M, int64_t D, int64_t F,
                                const uint32_t* W_gate, const float* beta_gate,
                                const uint32_t* W_up, const float* beta_up,
                                const uint32_t* W_down, const float* beta_down,
                                float* y, float* u, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* Decode engine                                                             */
/* ------------------------------------------------------------------------ */

/* Engines for the decode forward (M <= 64 tokens). */
enum {
    BL_ENGINE_AUTO = 0,          /* the library picks per shape (default): the CUDA-core GEMV
                                    for M <= 4, the swap-AB decode kernel for 5 <= M <= 16
                                    where it fits (for one problem of more than 8 tokens only
                                    while each CTA's rows fit one 128-lane tile), the tcgen05
                                    GEMM otherwise */
    BL_ENGINE_CUDA_CORES = 1,    /* M <= 64 on CUDA cores (masked byte dot products) */
    BL_ENGINE_TENSOR_CORES = 2,  /* M <= 16 on the swap-AB tcgen05 decode kernel where it
                                    fits (weight rows on the MMA's 128 lanes), else as AUTO */
    BL_ENGINE_CUDA_CORES_GENERAL = 3  /* as BL_ENGINE_CUDA_CORES, but one token also runs the
                                         general small-M kernel instead of the one-token
                                         streaming kernel */
};

/*
 * Selects the decode engine of every later forward call in this process
 * (bitlinear_forward, _fp, _fp_batch, _acc, _noalloc with M <= 64).  All
 * kernels compute the same integers and the same floats, bit for bit; the
 * choice only changes speed.  Not a feature of the pages: an
 * implementation switch, used by tests to check both engines.  Returns
 * BL_ERR_SHAPE for an unknown engine.  Takes effect for calls made after it
 * returns; not synchronised with calls made concurrently from other threads.
 */
bl_status bitlinear_set_decode_engine(int engine);

/* The engine last set (BL_ENGINE_AUTO initially). */
int bitlinear_get_decode_engine(void);

/* Kernel families of the forward. */
enum {
    BL_PATH_CUDA_CORES = 0,  /* CUDA-core GEMV (masked byte dot products) */
    BL_PATH_SWAP_AB = 1,     /* tcgen05 swap-AB decode kernel (weight rows on the MMA lanes) */
    BL_PATH_GEMM = 2         /* tcgen05 int8 GEMM (x_q rows on the MMA lanes) */
};

/*
 * Which kernel family bitlinear_forward / _fp / _acc would run for one
 * problem of M tokens, K input channels and N outputs on the current device
 * under the current engine, written to *path (a BL_PATH_* value).  An
 * implementation query, not a feature of the pages.  Errors: BL_ERR_NULL
 * (path null), BL_ERR_SHAPE (M < 1, N < 1, K < 64 or K % 64 != 0),
 * BL_ERR_DEVICE (no usable device).
 */
bl_status bitlinear_forward_path(int64_t M, int64_t N, int64_t K, int* path);

/* ------------------------------------------------------------------------ */
/* Diagnostics                                                               */
/* ------------------------------------------------------------------------ */

/*
 * Synchronises `stream`, then reads and clears the library's device error
 * word on the current device.  Returns BL_ERR_TIMEOUT if any kernel since the
 * last call gave up a bounded wait (the kernel then returned early and its
 * outputs are unspecified), BL_ERR_CUDA on a CUDA error, else BL_OK.
 */
bl_status bitlinear_device_status(void* stream);

/* Number of SMs of the current device as seen by the library (0 if none). */
int bitlinear_num_sms(void);

/*
 * Test hook of the bounded waits (no counterpart on the pages).  With
 * enable != 0, the next launch of the general small-M CUDA-core decode
 * kernel (M <= 4 tokens; with the engine BL_ENGINE_CUDA_CORES_GENERAL it
 * also runs one token) limits each wait of its first problem to about 10^5
 * SM cycles, and the weight producer of that problem's first CTA issues no
 * copies, so that CTA's consumers give up waiting for
 * data that never comes: the kernel raises the device error word and
 * returns (no copy is in flight, nothing hangs), that CTA's outputs are
 * unspecified, and the next bitlinear_device_status returns BL_ERR_TIMEOUT.
 * The request applies to one launch and then clears itself; enable == 0
 * withdraws it.  A launch recorded into a CUDA graph keeps it.  Always
 * returns BL_OK.
 */
bl_status bitlinear_test_expire_next_wait(int enable);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H */
