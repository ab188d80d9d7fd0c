/*
 * q8.h -- C ABI of the B200 (sm_100a) 8-bit quantized linear layer.
 *
 * The library computes the hot path of an 8-bit quantized nn.Linear:
 *   - per-output-channel weight quantization (asymmetric or symmetric INT8, FP8 E4M3);
 *   - dynamic per-token activation quantization (symmetric INT8 with row sums,
 *     or FP8 E4M3 with an upper-bound clip);
 *   - the W8A8 GEMM with INT32 / FP32 accumulation and a dequant epilogue;
 *   - the LLM.int8 mixed decomposition (outlier feature columns in fp16);
 *   - around it: activations with a static (calibrated) scale, smoothed
 *     activations (SmoothQuant-style per-column multipliers), and a W8A8 linear
 *     that re-quantizes its output to INT8 for the next layer;
 *   - group-wise 4-bit weights with one absmax scale per group of 32-128
 *     values along K (optionally with GGUF Q4_K-style quantized group scales),
 *     multiplied with 16-bit activations (W4A16);
 *   - the grouped FP8 rowwise linear of mixture-of-experts layers.
 *
 * Notation follows the pages' linear map Q = round(R / S) + Z, R = S (Q - Z):
 * `scale` is S, the dequant multiplier, and `zero_point` is Z, an integer held
 * in fp32.  Page short names used in the citations:
 *   [Fabric]   "8-Bit LLM Quantization with Lightning Fabric" (mlqm.cn)
 *   [CSDN]     "大模型量化技术" overview (devpress.csdn.net), sections 2.1-2.3
 *   [FBGEMM]   "Transformers FP8 (W8A8) 量化实战：基于 FBGEMM", sections 5.1-5.3, 6
 *   [LLM.int8] "Transformers 单 GPU 高效推理：bitsandbytes LLM.int8 8-bit 混合精度量化"
 *   [Xilyfe]   "大模型量化" (xilyfe.github.io): symmetric, asymmetric, INT32 accumulator,
 *              GGUF block quantization
 *
 * Conventions shared by every entry point
 *   Layout      all matrices are row-major 2-D: X is M x K (tokens x features),
 *               W is N x K (out x in, the nn.Linear layout of [FBGEMM] 5.1),
 *               Y is M x N.  Leading dimensions are in elements.  Callers flatten
 *               leading batch dims first ([FBGEMM] 5.2-5.3: x.view(-1, K), then
 *               the result is viewed back to (*x.shape[:-1], -1)).
 *   Memory      every pointer is DEVICE memory owned by the caller, unless a
 *               parameter says "host".  The library allocates nothing: scratch
 *               comes from the caller's `workspace` (see q8_workspace_size).
 *   Streams     every call is asynchronous on `stream` (a cudaStream_t; NULL is
 *               the legacy default stream) and never synchronizes the host,
 *               except q8_get_device_status.
 *   Sizes       K % 32 == 0, N % 16 == 0, M >= 0; M, N, K <= 2^31 - 1;
 *               INT8 GEMMs need K <= 32768 (INT32 accumulator bound).
 *               M == 0 is a valid empty call that launches nothing.
 *   Alignment   every pointer 16-byte aligned; every leading dimension a
 *               multiple of 16 bytes.
 *   Values      inputs must be finite; NaN and Inf inputs give unspecified codes.
 *   Rounding    round-half-to-even everywhere; q = rne(fl32(x / S)) for the
 *               IEEE fp32 quotient (the kernels reach its rounding without a
 *               division per element), so codes are bit-exact with a scalar
 *               reference; S is floored at 1e-8 ([Xilyfe] QuantConfig eps).
 *   Errors      every call returns a q8_status and never prints, throws or
 *               aborts.  Arguments are validated on the host before anything is
 *               launched, so an error return means nothing was enqueued.
 *               Device-side waits are bounded (about one second); a wait that
 *               runs out records Q8_ERR_DEVICE_TIMEOUT in a per-device status
 *               word read by q8_get_device_status.
 *   Hardware    compute capability 10.0 (B200, sm_100a) only; anything else
 *               returns Q8_ERR_UNSUPPORTED_ARCH after argument validation.
 */
#ifndef Q8_H_
#define Q8_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define Q8_VERSION 8

/* Same object as cudaStream_t. */
typedef struct CUstream_st *q8_stream_t;

typedef enum {
    Q8_OK = 0,
    Q8_ERR_NULL = 1,             /* a required pointer is NULL */
    Q8_ERR_SHAPE = 2,            /* a size or leading dimension is out of range */
    Q8_ERR_ALIGN = 3,            /* a pointer or leading dimension is not 16-byte aligned */
    Q8_ERR_DTYPE = 4,            /* unsupported dtype, or dtypes that do not fit together */
    Q8_ERR_SCHEME = 5,           /* unsupported scheme, or scheme / code dtype mismatch */
    Q8_ERR_UNSUPPORTED_ARCH = 6, /* the current device is not compute capability 10.0 */
    Q8_ERR_LAUNCH = 7,           /* a kernel launch failed */
    Q8_ERR_DEVICE_TIMEOUT = 8,   /* a bounded device wait ran out (q8_get_device_status) */
    Q8_ERR_WORKSPACE = 9,        /* workspace NULL or smaller than q8_workspace_size */
    Q8_ERR_CUDA = 10             /* another CUDA runtime error (no device, bad stream, ...) */
} q8_status;

typedef enum {
    Q8_S8 = 0,    /* int8 codes */
    Q8_U8 = 1,    /* uint8 codes (asymmetric weights stored as q + 128) */
    Q8_E4M3 = 2,  /* OCP FP8 E4M3FN codes (max 448, no infinities) */
    Q8_F16 = 3,   /* IEEE binary16 */
    Q8_BF16 = 4,  /* bfloat16 */
    Q8_F32 = 5,
    Q8_S32 = 6
} q8_dtype;

typedef enum {
    Q8_ASYM_INT8 = 0, /* per-row min-max, S = (max - min)/255, Z = rne(-min/S) - 128 */
    Q8_SYM_INT8 = 1,  /* per-row absmax, S = absmax/127, Z = 0, codes in [-127, 127] */
    Q8_FP8_E4M3 = 2   /* per-row absmax, S = absmax/448, codes E4M3 saturating */
} q8_scheme;

/* A quantized weight: N x K codes (row stride `ld` elements) with one scale per
 * row and, for asymmetric codes, one zero point per row.  For Q8_U8 codes the
 * zero point is in the uint8 convention (Z + 128), so S (q - zero_point) is
 * the dequantized value in both conventions. */
typedef struct {
    const void *codes;
    q8_dtype code_dtype;          /* Q8_S8, Q8_U8 or Q8_E4M3 */
    const float *scale;           /* [n] */
    const float *zero_point;      /* [n] integer-valued; NULL for symmetric / FP8 */
    int64_t n, k, ld;
} q8_weight;

/* A quantized activation: M x K codes with one scale per row and, for INT8,
 * the int32 row sums of the codes (needed when the weight has a zero point). */
typedef struct {
    const void *codes;
    q8_dtype code_dtype;          /* Q8_S8 or Q8_E4M3 */
    const float *scale;           /* [m] */
    const int32_t *rowsum;        /* [m]; may be NULL when the weight has no zero point */
    int64_t m, k, ld;
} q8_act;

/*
 * Per-output-channel weight quantization, one row of W at a time.
 * [Fabric] 2.1, 2.3 and 3.3 (one scale and zero point per output row);
 * [Xilyfe] asymmetric section (s = 255/(alpha-beta), z = round(-s beta) - 128)
 * and symmetric section (s = 127/alpha); [CSDN] 2.3 min-max calibration;
 * [FBGEMM] 5.1 (e4m3 weight, fp32 weight_scale per output channel).
 *
 *   W           device, n x k, w_dtype Q8_F16, Q8_BF16 or Q8_F32, row stride ldw.
 *   scheme      Q8_ASYM_INT8 (code_dtype Q8_S8 or Q8_U8), Q8_SYM_INT8 (Q8_S8),
 *               Q8_FP8_E4M3 (Q8_E4M3).
 *   codes       device, n x k output, row stride k.
 *   scale       device [n] output.
 *   zero_point  device [n] output for Q8_ASYM_INT8 (required); ignored (may be
 *               NULL) for the other schemes.
 * Asymmetric, per row with beta = min, alpha = max:
 *   S = max(fl32(fl32(alpha - beta) / 255), 1e-8);
 *   Z = clamp(rne(fl32(-beta / S)) - 128, -128, 127);
 *   q = clamp(rne(fl32(w / S)) + Z, -128, 127)   (stored + 128 for Q8_U8, Z too).
 * Symmetric: S = max(fl32(absmax / 127), 1e-8); q = clamp(rne(fl32(w / S)), -127, 127).
 * FP8: S = max(fl32(absmax / 448), 1e-8); q = e4m3_rne_satfinite(fl32(w / S)).
 */
q8_status q8_quantize_weight(const void *W, q8_dtype w_dtype, int64_t n, int64_t k,
                             int64_t ldw, q8_scheme scheme, q8_dtype code_dtype,
                             void *codes, float *scale, float *zero_point,
                             q8_stream_t stream);

/*
 * Dequantize a weight back to floating point for debugging, out = S (q - Z)
 * ([Fabric] 3.3 dequantize_weight; [Xilyfe] "量化是什么": r = S (q - Z)).
 * fp32 order: d = fl32(q - Z), v = fl32(S * d), then RNE to out_dtype.
 *   out   device, w->n x w->k, out_dtype Q8_F32, Q8_F16 or Q8_BF16, row stride w->k.
 */
q8_status q8_dequantize_weight(const q8_weight *w, q8_dtype out_dtype, void *out,
                               q8_stream_t stream);

/*
 * Dynamic per-token activation quantization, every call.
 * [Xilyfe] symmetric section and dynamic-quantization paragraph; [FBGEMM] 5.2
 * (quantize_fp8_per_row with the activation_scale_ub clip) and 6 (ub 1200.0).
 *
 *   X        device, m x k, x_dtype Q8_F16, Q8_BF16 or Q8_F32, row stride ldx.
 *   scheme   Q8_SYM_INT8: S = max(fl32(absmax/127), 1e-8),
 *              q = clamp(rne(fl32(x/S)), -127, 127), codes int8;
 *            Q8_FP8_E4M3: alpha = min(absmax, clip_ub) when clip_ub > 0,
 *              S = max(fl32(alpha/448), 1e-8), q = e4m3_rne_satfinite(fl32(x/S)).
 *   clip_ub  FP8 only; <= 0 means no clip.
 *   codes    device, m x k output (int8 or e4m3), row stride k.
 *   scale    device [m] output.
 *   rowsum   device [m] int32 output, sum_k q (INT8 only; may be NULL).
 */
q8_status q8_quantize_act(const void *X, q8_dtype x_dtype, int64_t m, int64_t k,
                          int64_t ldx, q8_scheme scheme, float clip_ub, void *codes,
                          float *scale, int32_t *rowsum, q8_stream_t stream);

/*
 * Static activation quantization with a calibrated per-tensor scale: the scale
 * is computed once, offline, from a calibration pass and applied to every call
 * ([Xilyfe] the paragraph on static quantization, 静态量化).  Symmetric INT8,
 * q = clamp(rne(fl32(x / static_scale)), -127, 127): inputs beyond
 * 127 * static_scale saturate.  The output is a q8_act like the dynamic one.
 *   X             device, m x k, Q8_F16 / Q8_BF16 / Q8_F32, row stride ldx.
 *   static_scale  > 0 and finite, else Q8_ERR_SCHEME.
 *   codes         device, m x k int8 output, row stride k.
 *   scale         device [m] output, every entry static_scale.
 *   rowsum        device [m] int32 output, sum_k q (may be NULL).
 */
q8_status q8_quantize_act_static(const void *X, q8_dtype x_dtype, int64_t m, int64_t k,
                                 int64_t ldx, float static_scale, void *codes, float *scale,
                                 int32_t *rowsum, q8_stream_t stream);

/*
 * Dynamic per-token INT8 quantization of a smoothed activation ([Xilyfe]
 * algorithm list, SmoothQuant: outlier channels of the activation are moved
 * onto the weight, which leaves X W^T unchanged and makes the activation easy
 * to quantize).  Column j is multiplied by mult[j] = RN(1 / s_j) before the
 * quantizer of q8_quantize_act (Q8_SYM_INT8) runs: xs = fl32(x * mult[j]),
 * S = max(fl32(max|xs| / 127), 1e-8), q = clamp(rne(fl32(xs / S)), -127, 127).
 * The smoothing factors s_j are chosen offline; the weight is smoothed offline
 * too (W[:, j] * s_j) and quantized with q8_quantize_weight.
 *   mult     device [k] float, 16-byte aligned.
 *   others   as q8_quantize_act with Q8_SYM_INT8.
 */
q8_status q8_quantize_act_smooth(const void *X, q8_dtype x_dtype, int64_t m, int64_t k,
                                 int64_t ldx, const float *mult, void *codes, float *scale,
                                 int32_t *rowsum, q8_stream_t stream);

/*
 * LLM.int8 outlier detection fused with the regular stream's quantization
 * ([LLM.int8] 核心思想 and BitsAndBytesConfig: llm_int8_threshold = 6.0).
 * A feature column k is an outlier when some token has |X[m, k]| > threshold
 * (strictly); threshold <= 0 turns the decomposition off.  Then, per token,
 * alpha is the absmax over the non-outlier columns and the INT8 codes of
 * outlier columns are 0 (the regular stream is "the rest").
 *
 *   X             device, m x k fp16 (Q8_F16), row stride ldx.
 *   codes         device, m x k int8 output, row stride k.
 *   scale         device [m] output;  rowsum device [m] int32 output.
 *   mask          device [k] uint8 output: 1 for outlier columns.
 *   idx           device [k] int32 output: outlier columns ascending in
 *                 idx[0 .. *count); entries past *count are unspecified.
 *   count         device int32 output (stays on the device).
 *   x_outlier     device, m x ldo fp16 output: x_outlier[m, j] = X[m, idx[j]]
 *                 for j < *count and 0 for count <= j < round_up(count, 64);
 *                 may be NULL.  ldo >= round_up(k, 64) and a multiple of 8.
 * The column pass reads all m rows, so the outlier set depends on the batch.
 */
q8_status q8_outlier_quantize_act(const void *X, q8_dtype x_dtype, int64_t m, int64_t k,
                                  int64_t ldx, float threshold, void *codes, float *scale,
                                  int32_t *rowsum, uint8_t *mask, int32_t *idx,
                                  int32_t *count, void *x_outlier, int64_t ldo,
                                  q8_stream_t stream);

/*
 * W8A8 linear: Y = dequant(x) dequant(w)^T (+ bias), bf16 out.
 * INT8 ([Xilyfe] INT32 accumulator section; [CSDN] 2.1 quantized matmul read
 * with R = S (Q - Z)):
 *   acc[m, n] = sum_k xq[m, k] wq[n, k]                  (tensor cores, int32)
 *   y = fl32(fl32(fl32(acc - Z[n] rowsum[m]) * Sx[m]) * Sw[n]);  y = fl32(y + bias[n])
 * FP8 ([FBGEMM] 5.3 f8f8bf16_rowwise, then + bias):
 *   acc = sum_k e4m3(xq) e4m3(wq) (tensor cores, fp32);  y = fl32(fl32(acc*Sx)*Sw) (+bias)
 * Y[m, n] = bf16_rne(y).
 *
 *   x          INT8 (Q8_S8) with x->rowsum required when w->zero_point is set,
 *              or FP8 (Q8_E4M3); x->k == w->k.
 *   w          Q8_S8 / Q8_U8 (with or without zero point) for INT8 x;
 *              Q8_E4M3 for FP8 x.
 *   bias       device [n] fp32, or NULL.
 *   Y          device, m x n bf16 output, row stride ldy >= n.
 *   acc_debug  device, m x n int32 (INT8) or fp32 (FP8) raw accumulator
 *              output (row stride n), or NULL.
 *   workspace  unused by this call today; pass q8_workspace_size(Q8_OP_LINEAR_W8A8, ...)
 *              bytes (currently 0; NULL accepted).
 * Launch overlap: the quantize and GEMM kernels are launched with
 * programmatic dependent launch, and each waits for the kernel before it
 * before reading anything that kernel may write.  The one exception is the
 * weight: every GEMM kernel requests its first weight slices before that
 * wait, so when the kernel right before it triggers programmatic launch early
 * (this library's activation quantizers and LLM.int8 row pass do), the weight
 * loads overlap that kernel and the one before it.  The weight must therefore
 * not be written by a kernel that triggers programmatic launch early
 * (griddepcontrol.launch_dependents) and runs just before the GEMM or its
 * quantizer.  This library's weight quantizers do not trigger, so
 * quantize_weight followed by any sequence of these calls is safe.
 */
q8_status q8_linear_w8a8(const q8_act *x, const q8_weight *w, const float *bias, void *Y,
                         int64_t ldy, void *acc_debug, void *workspace, size_t ws_bytes,
                         q8_stream_t stream);

/*
 * INT8 W8A8 linear whose output is re-quantized to INT8 codes for the next
 * layer instead of written as bf16 ([Xilyfe] 量化对象 section: after the INT32
 * accumulation the result is scaled back into INT8 before it is passed on).
 * y is the fp32 value q8_linear_w8a8 would round to bf16 (dequant epilogue and
 * bias); the output is clamp(rne(fl32(y / out_scale)), -127, 127), with
 * out_scale the next layer's static input scale.
 *   x, w, bias   as q8_linear_w8a8, INT8 codes only (Q8_ERR_DTYPE for E4M3).
 *   out_scale    > 0 and finite, else Q8_ERR_SCHEME.
 *   Yq           device, m x w->n int8 output, row stride ldy (ldy % 16 == 0).
 *   acc_debug    as q8_linear_w8a8.
 * The launch-overlap rule of q8_linear_w8a8 applies.
 */
q8_status q8_linear_w8a8_requant(const q8_act *x, const q8_weight *w, const float *bias,
                                 float out_scale, void *Yq, int64_t ldy, void *acc_debug,
                                 q8_stream_t stream);

/* A group-wise 4-bit weight: n x k values, one fp32 scale per group of
 * `group` consecutive values along K ([CSDN] 2.2 granularity table: one scale
 * per group of 64-128 parameters; [Xilyfe] GGUF section: each block of a row
 * has its own absmax scale).  Dequantized value: scale * (nibble - 8).
 *   codes   n x k/2 bytes, row stride ld bytes (ld >= k/2, ld % 16 == 0);
 *           byte j of a row holds element 2j in its low nibble and element
 *           2j+1 in its high nibble, each as q + 8 with q in [-7, 7].
 *   scale   (k / group) x n fp32, GROUP-major: scale[j * n + r] belongs to row
 *           r, elements j*group .. j*group + group - 1.
 *   group   32, 64 or 128; k % group == 0. */
typedef struct {
    const void *codes;
    const float *scale;
    int64_t n, k, ld;
    int32_t group;
} q8_weight_g4;

/*
 * Group-wise symmetric 4-bit weight quantization ([Xilyfe] GGUF section:
 * s = absmax / 7 per block, codes round(w / s); [CSDN] 2.2 group granularity).
 * For each row r and group j: S = fl32(max |w| / 7), floored at 1e-8;
 * q = clamp(rne(fl32(w / S)), -7, 7).  Bit-exact with a scalar reference.
 *
 *   W       device, n x k, Q8_F16 or Q8_BF16, row stride ldw (elements).
 *   group   32, 64 or 128 (Q8_ERR_SCHEME otherwise); k % group == 0 and
 *           k % 32 == 0, n % 16 == 0 (Q8_ERR_SHAPE).
 *   codes   device output, n x k/2 bytes, row stride ldc bytes (ldc >= k/2,
 *           ldc % 16 == 0), layout of q8_weight_g4.
 *   scale   device output, (k / group) x n fp32, group-major.
 * One launch; offline (once per weight).
 */
q8_status q8_quantize_weight_g4(const void *W, q8_dtype w_dtype, int64_t n, int64_t k,
                                int64_t ldw, int32_t group, void *codes, int64_t ldc,
                                float *scale, q8_stream_t stream);

/*
 * GGUF Q4_K-style weights ([Xilyfe] GGUF section, Q4_K simulation): groups of
 * 32 along K (sub-blocks) quantized as q8_quantize_weight_g4 with group 32,
 * whose scales are quantized again per super block of 8 sub-blocks (256
 * values): s_super = fl32(max s_sub / 15), sub-scale codes
 * c = clamp(rne(fl32(s_sub / s_super)), 0, 15).  The weight codes come from the
 * unquantized sub-block scale (the page's order); a sub-block is dequantized
 * with fl32(s_super * c).  Bit-exact with a scalar reference.
 *
 *   W            device, n x k, Q8_F16 or Q8_BF16, row stride ldw; k % 256 == 0,
 *                n % 16 == 0 (Q8_ERR_SHAPE).
 *   codes, ldc   device output, as q8_quantize_weight_g4.
 *   scale        device output, (k / 32) x n fp32, group-major: the effective
 *                scales fl32(s_super * c), so {codes, scale, group = 32} is a
 *                q8_weight_g4 for q8_linear_w4a16.
 *   sub_codes    device output, (k / 64) x n bytes: byte [j][r] holds the codes
 *                of sub-blocks 2j (low nibble) and 2j+1 (high nibble) of row r.
 *   super_scale  device output, (k / 256) x n fp32.
 * sub_codes and super_scale are the compact stored form (1 byte of scale per
 * 32 weights instead of 4); q8_expand_q4k_scales rebuilds `scale` from them.
 */
q8_status q8_quantize_weight_q4k(const void *W, q8_dtype w_dtype, int64_t n, int64_t k,
                                 int64_t ldw, void *codes, int64_t ldc, float *scale,
                                 uint8_t *sub_codes, float *super_scale, q8_stream_t stream);

/*
 * scale[j * n + r] = fl32(super_scale[(j / 8) * n + r] * c_j) for the compact
 * Q4_K scales written by q8_quantize_weight_q4k (layouts as there); the result
 * is bit-identical to the `scale` output of that call.  k % 256 == 0,
 * n % 16 == 0.  One launch.
 */
q8_status q8_expand_q4k_scales(const uint8_t *sub_codes, const float *super_scale, int64_t n,
                               int64_t k, float *scale, q8_stream_t stream);

/*
 * W4A16 linear: Y = X W~^T (+ bias), W~ the group-wise 4-bit weight brought
 * back to the activation's 16-bit format.  The weight of each K slice is
 * dequantized in shared memory, w~ = round16(fl32(S * q)), and multiplied on
 * the tensor cores with fp32 accumulation; y = fl32(y + bias[n]); Y = bf16(y).
 * The fp32 accumulation order is not specified (results agree with an exact
 * sum of the same w~ within the fp32 accumulation bound).
 *
 *   X       device, m x k activations, Q8_BF16 or Q8_F16 (Q8_ERR_DTYPE
 *           otherwise), row stride ldx (elements, 16-byte multiple).
 *   w       group-wise weight with w->k == k (Q8_ERR_SHAPE otherwise).
 *   bias    device [w->n] fp32, or NULL.
 *   Y       device, m x w->n bf16, row stride ldy (ldy % 8 == 0).
 * One launch.  It may start before the previous kernel on `stream` has ended
 * (programmatic dependent launch) and waits for it before reading X or
 * writing Y.
 */
q8_status q8_linear_w4a16(const void *X, q8_dtype x_dtype, int64_t m, int64_t k, int64_t ldx,
                          const q8_weight_g4 *w, const float *bias, void *Y, int64_t ldy,
                          q8_stream_t stream);

/*
 * Grouped FP8 rowwise linear of a mixture-of-experts layer ([FBGEMM] 5.4,
 * Llama4 experts: the experts' FP8 weights are stored together with per-row
 * scales, and each expert's tokens are quantized and multiplied with
 * f8f8bf16_rowwise on their own).  Tokens are sorted by expert: rows
 * offsets[e] .. offsets[e+1]-1 of x use expert e, whose weight is rows
 * e*n .. e*n+n-1 of w (n = w->n / num_experts), with the same scales and bias
 * rows.  Per token and channel: acc = sum_k e4m3 x e4m3 (fp32),
 * y = fl32(fl32(acc * Sx[m]) * Sw[e*n + j]) (+ bias[e*n + j]), Y = bf16(y).
 * Quantize the sorted activations with q8_quantize_act(Q8_FP8_E4M3): its
 * per-token scales are the same whether taken per expert or over all tokens.
 *
 *   x            E4M3 activation codes, x->m tokens sorted by expert.
 *   w            E4M3 weights of all experts stacked, w->n = num_experts * n,
 *                per-row scales; n % 16 == 0.
 *   num_experts  1 .. 4096; ceil(x->m / 128) + num_experts <= 65535.
 *   offsets      device int32 [num_experts + 1], non-decreasing, offsets[0] = 0,
 *                offsets[num_experts] = x->m (typically the previous kernel's
 *                routing result).  Out-of-range values are clamped to
 *                [0, x->m], so no call writes outside Y; rows no expert
 *                covers are left unwritten.
 *   bias         device fp32 [w->n] (per expert, stacked), or NULL.
 *   Y            device, x->m x n bf16 (sorted token order), row stride ldy
 *                (ldy % 8 == 0).
 * One launch; the fp32 accumulation order is not specified (the FP8 bound of
 * q8_linear_w8a8 applies).  It may start before the previous kernel on
 * `stream` has ended and waits for it before reading anything.
 */
q8_status q8_linear_fp8_grouped(const q8_act *x, const q8_weight *w, int64_t num_experts,
                                const int32_t *offsets, const float *bias, void *Y, int64_t ldy,
                                q8_stream_t stream);

/*
 * Dynamic per-token activation quantization and the W8A8 linear in one call:
 * the same results, bit for bit, as q8_quantize_act(X, act_scheme, clip_ub)
 * followed by q8_linear_w8a8 ([Xilyfe] dynamic quantization: the activation
 * scale is computed from each call's input; [FBGEMM] 5.2-5.3: quantize the
 * input per row, then the rowwise GEMM, on every forward).
 *
 *   X            device, m x k, Q8_F16 / Q8_BF16 / Q8_F32, row stride ldx.
 *   act_scheme   Q8_SYM_INT8 with an INT8 weight (Q8_S8 / Q8_U8), or
 *                Q8_FP8_E4M3 with an E4M3 weight; clip_ub as q8_quantize_act.
 *   act_codes    device m x k output codes (row stride k), act_scale [m] and,
 *   act_scale,   for INT8, act_rowsum [m]: the quantized activation, written as
 *   act_rowsum   q8_quantize_act writes it (required).
 *   acc_debug    as q8_linear_w8a8.
 * Two launches: the quantizer lets the GEMM start early (programmatic
 * dependent launch), so the GEMM's prologue and weight loads overlap the
 * quantization.  The launch-overlap rule of q8_linear_w8a8 applies.
 */
q8_status q8_linear_w8a8_dynamic(const void *X, q8_dtype x_dtype, int64_t m, int64_t k,
                                 int64_t ldx, q8_scheme act_scheme, float clip_ub,
                                 const q8_weight *w, const float *bias, void *Y, int64_t ldy,
                                 void *act_codes, float *act_scale, int32_t *act_rowsum,
                                 void *acc_debug, q8_stream_t stream);

/*
 * LLM.int8 mixed-decomposition linear ([LLM.int8] 核心思想; BitsAndBytesConfig
 * llm_int8_threshold, llm_int8_has_fp16_weight).  One call runs
 * q8_outlier_quantize_act on X, the INT8 GEMM of the regular stream, and the
 * fp16 GEMM of the outlier columns, merged before rounding:
 *   y16[m, n] = sum_{j < count} X[m, idx[j]] W16[n, idx[j]]   (fp16 in, fp32 acc)
 *   y = fl32(y_int8 + y16);  y = fl32(y + bias[n]);  Y = bf16_rne(y)
 * with y_int8 the INT8 epilogue above without bias.
 *
 *   X              device, m x k fp16 (Q8_F16), row stride ldx.
 *   w              INT8 weight (Q8_S8 or Q8_U8, zero point optional).
 *   W16            device n x k fp16 original weight, row stride k, when the
 *                  caller keeps it (llm_int8_has_fp16_weight); NULL (the default)
 *                  uses fp16_rne(fl32(S[n] * fl32(q - Z))) for the outlier columns.
 *   threshold      6.0 by default; <= 0 turns the decomposition off.
 *   bias, Y, ldy   as q8_linear_w8a8.
 *   outlier_mask   device [k] uint8 output, or NULL.
 *   outlier_count  device int32 output, or NULL.
 *   acc_debug      device m x n int32 raw INT8 accumulator, or NULL.
 *   y16_debug      device m x n fp32 outlier-stream result, or NULL.
 *   workspace      device scratch of at least
 *                  q8_workspace_size(Q8_OP_LINEAR_INT8_MIXED, m, n, k) bytes,
 *                  256-byte aligned; contents need no initialization.
 */
q8_status q8_linear_int8_mixed(const void *X, q8_dtype x_dtype, int64_t m, int64_t k,
                               int64_t ldx, const q8_weight *w, const void *W16,
                               float threshold, const float *bias, void *Y, int64_t ldy,
                               uint8_t *outlier_mask, int32_t *outlier_count,
                               int32_t *acc_debug, float *y16_debug, void *workspace,
                               size_t ws_bytes, q8_stream_t stream);

/*
 * q8_linear_int8_mixed without a caller workspace, for callers that cannot
 * allocate device memory: an engine that plans all of its device memory up
 * front and forbids allocation while serving, a plain C caller with no device
 * allocator, or code running where cudaMalloc may not be called.  (The pages
 * have no counterpart: this is an interface convenience of this library.)
 *
 * Same arguments and results as q8_linear_int8_mixed, minus workspace and
 * ws_bytes.  The scratch is one static device array inside the library, of
 * Q8_NOALLOC_SCRATCH_BYTES (64 MiB); every GPU that loads the library's module
 * holds it until the process exits.  This call allocates nothing and calls no
 * allocating routine.
 *   Limit     q8_workspace_size(Q8_OP_LINEAR_INT8_MIXED, m, w->n, k) must not
 *             exceed Q8_NOALLOC_SCRATCH_BYTES (e.g. m <= 512 at n = k = 4096);
 *             larger sizes return Q8_ERR_SHAPE before anything is launched.
 *   Set-up    the first call on each device looks up the array's device
 *             address (cudaGetSymbolAddress, with that device current) and
 *             caches it; make that first call before any stream capture.
 *             cudaDeviceReset destroys the array with the context, and the
 *             cached address with it: do not call this entry point on a
 *             device after resetting it in the same process.
 *   Sharing   every call on a device uses the same scratch, which keeps the
 *             last call's contents (nothing in it needs to start at zero).
 *             Calls whose executions overlap on the GPU (other streams, other
 *             threads) race on it: serialize them.
 */
#define Q8_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

q8_status q8_linear_int8_mixed_noalloc(const void *X, q8_dtype x_dtype, int64_t m, int64_t k,
                                       int64_t ldx, const q8_weight *w, const void *W16,
                                       float threshold, const float *bias, void *Y, int64_t ldy,
                                       uint8_t *outlier_mask, int32_t *outlier_count,
                                       int32_t *acc_debug, float *y16_debug,
                                       q8_stream_t stream);

enum { Q8_OP_LINEAR_W8A8 = 0, Q8_OP_LINEAR_INT8_MIXED = 1 };

/* Bytes of device workspace an operation needs for these sizes (host function,
 * no device access).  The mixed operation sizes its outlier buffers for every
 * column being an outlier, so no call can overflow them.  Returns 0 for an
 * operation that needs none or for negative sizes, and SIZE_MAX when a size
 * exceeds 2^31 - 1 (no such call is valid). */
size_t q8_workspace_size(int op, int64_t m, int64_t n, int64_t k);

/* Static, NUL-terminated description of a status code (host). */
const char *q8_status_string(q8_status s);

/* Waits for `stream`, then reads the current device's status word into *out
 * (host pointer): Q8_OK, or the first device-side error recorded since the
 * last clear (Q8_ERR_DEVICE_TIMEOUT). */
q8_status q8_get_device_status(int32_t *out, q8_stream_t stream);

/* Resets the current device's status word to Q8_OK (enqueued on `stream`). */
q8_status q8_clear_device_status(q8_stream_t stream);

/*
 * Self-test of the device-side failure detection described under "Errors"
 * above (the pages have no counterpart: it tests this library's own
 * bounded waits).  Enqueues on `stream` one CTA with the GEMM kernels' roles
 * (a TMA producer warp, an MMA warp and four epilogue warps sharing an abort
 * flag, with tensor memory allocated) whose producer waits on a barrier that
 * nothing ever arrives on, bounded by `limit_us` microseconds instead of the
 * usual second.  When the wait runs out the kernel records
 * Q8_ERR_DEVICE_TIMEOUT in the current device's status word, the other roles
 * leave their waits on the abort flag, the CTA frees its tensor memory and
 * returns: nothing faults or hangs and the context stays usable.  Read the
 * result with q8_get_device_status and reset it with q8_clear_device_status.
 * Returns Q8_ERR_SHAPE unless 1 <= limit_us <= 1000000, else Q8_OK once the
 * kernel is enqueued (or the q8_device_check status).
 */
q8_status q8_selftest_wait_timeout(int32_t limit_us, q8_stream_t stream);

/* Q8_OK when the current device can run this library, else
 * Q8_ERR_UNSUPPORTED_ARCH or Q8_ERR_CUDA (host). */
q8_status q8_device_check(void);

/*
 * Host-side fault injection, for testing a caller's error handling (host).
 * Arms a one-shot failure: after `skip` more calls that pass their argument
 * validation, the next such call returns `code` without enqueuing anything;
 * then the hook is disarmed.  Calls that fail validation do not count.
 * Applies to every entry point that launches work (not to q8_device_check,
 * q8_get_device_status or q8_clear_device_status).  code = Q8_OK disarms.
 * Returns Q8_ERR_SCHEME for a code that is not a q8_status, Q8_ERR_SHAPE for
 * skip < 0.  Process-wide; safe to call from any thread.
 */
q8_status q8_inject_failure(q8_status code, int32_t skip);

/* Q8_VERSION of the built library (host). */
int q8_version(void);

#ifdef __cplusplus
}
#endif

#endif /* Q8_H_ */
