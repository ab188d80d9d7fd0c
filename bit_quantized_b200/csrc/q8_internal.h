// Host-side declarations shared by the library's translation units.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/q8.h"

namespace q8 {

// Device address of the current device's status word (set up once per device).
int* device_status_ptr();

// ---- quantize kernels (q8_quant.cu)
enum RowOp { kOpActInt8 = 0, kOpActFp8 = 1, kOpWeightAsym = 2, kOpWeightSym = 3, kOpWeightFp8 = 4,
             kOpActInt8Static = 6, kOpActInt8Smooth = 7 };

struct RowQuantArgs {
    const void* src;       // rows x k input (f16 / bf16 / f32)
    q8_dtype src_dtype;
    int64_t rows, k, ld;   // ld in elements
    int op;                // RowOp
    bool codes_u8;         // asymmetric weights stored as uint8 (q + 128)
    float clip_ub;         // fp8 activations: > 0 clips the row absmax
    float static_scale;    // kOpActInt8Static: the calibrated scale (> 0)
    const float* mult;     // kOpActInt8Smooth: [k] per-column multipliers (1 / smoothing factor)
    const uint8_t* skip;   // [k] columns left out (LLM.int8 outliers); may be null
    void* codes;           // rows x k, row stride k
    float* scale;          // [rows]
    float* zero_point;     // [rows] or null
    int32_t* rowsum;       // [rows] or null
    // LLM.int8 (only with skip): the kernel ranks the outlier columns itself
    // (a block-wide scan of the mask) and writes the ascending column list and
    // the count (outputs), then gathers the outlier columns of X (rows x ldo
    // fp16, zero-padded to a multiple of 64) and, when w_rows > 0, of the
    // weight (w_rows x ldo fp16: W16's columns, or S (q - Z) rounded to fp16).
    int32_t* outlier_idx;
    int32_t* outlier_count;
    __half* x_outlier;     // or null
    int64_t ldo;
    int64_t w_rows;        // 0: no weight gather
    const void* w_codes;   // w_rows x w_ld int8 / uint8 codes
    bool w_codes_u8;
    int64_t w_ld;          // codes' (or W16's) leading dimension
    const float* w_scale;
    const float* w_zero;   // or null
    const __half* w16;     // original fp16 weight (has_fp16_weight), or null
    __half* w_outlier;     // w_rows x ldo
};

cudaError_t launch_row_quant(const RowQuantArgs& a, cudaStream_t s);

// Outlier mask of an LLM.int8 call: mask[c] = 1 for the columns c where some
// row has |x| > threshold (none when threshold <= 0).
cudaError_t launch_outlier_columns(const void* X, q8_dtype dt, int64_t m, int64_t k, int64_t ldx,
                                   float threshold, uint8_t* mask, cudaStream_t s);

cudaError_t launch_dequant(const q8_weight& w, q8_dtype out_dtype, void* out, cudaStream_t s);

// ---- GEMMs (q8_gemm.cu)
struct LinearArgs {
    int64_t m, n, k;
    const void* a_codes;  int64_t lda;     // activations m x k
    const void* b_codes;  int64_t ldb;     // weights n x k
    int kind;                              // 0: int8 x int8, 1: int8 x uint8, 2: e4m3 x e4m3
    const float* sx;
    const int32_t* rowsum;                 // null when zw is null
    const float* sw;
    const float* zw;                       // null: no zero point
    const float* bias;
    __nv_bfloat16* y;  int64_t ldy;
    int8_t* yq;  float out_scale;          // non-null yq: int8 output codes (requantized), y unused
    void* acc_debug;                       // m x n (row stride n), or null
    // LLM.int8 outlier stream (all null for plain W8A8)
    const __half* xo; int64_t ldxo;        // m x ldxo fp16 gathered outlier columns
    const __half* wo; int64_t ldwo;        // n x ldwo fp16 outlier weight columns
    const int32_t* outlier_count;          // device
    int64_t k16_cap;                       // columns the outlier buffers hold
    float* y16_debug;                      // m x n, or null
};

q8_status launch_linear(const LinearArgs& a, cudaStream_t s);

// ---- group-wise 4-bit weights (q8_w4.cu)
cudaError_t launch_group_quant(const void* W, q8_dtype dt, int64_t n, int64_t k, int64_t ldw,
                               int group, uint8_t* codes, int64_t ldc, float* scale,
                               cudaStream_t s);

cudaError_t launch_q4k_quant(const void* W, q8_dtype dt, int64_t n, int64_t k, int64_t ldw,
                             uint8_t* codes, int64_t ldc, float* scale, uint8_t* sub_codes,
                             float* super_scale, cudaStream_t s);
cudaError_t launch_q4k_expand(const uint8_t* sub_codes, const float* super_scale, int64_t n,
                              int64_t k, float* scale, cudaStream_t s);

struct W4Args {
    const void* x; bool x_bf16;            // m x k activations (bf16 or fp16), row stride ldx
    int64_t m, k, ldx;
    const void* codes; int64_t ldc;        // n x k/2 packed nibbles (q + 8), row stride ldc bytes
    const float* scale;                    // (k / group) x n, group-major
    int64_t n;
    int group;                             // 32, 64 or 128
    const float* bias;
    __nv_bfloat16* y; int64_t ldy;
};

q8_status launch_w4a16(const W4Args& a, cudaStream_t s);

// ---- grouped FP8 GEMM for mixture-of-experts layers (q8_moe.cu)
struct MoeArgs {
    int64_t m, k;                          // tokens sorted by expert, reduction depth
    const void* x_codes; int64_t ldx;      // m x k e4m3, row stride ldx bytes
    const float* sx;                       // [m]
    int64_t experts, n;                    // experts, output channels per expert
    const void* w_codes; int64_t ldw;      // experts*n x k e4m3, row stride ldw bytes
    const float* sw;                       // [experts * n]
    const int32_t* offsets;                // device [experts + 1]
    const float* bias;                     // [experts * n] or null
    __nv_bfloat16* y; int64_t ldy;
};

q8_status launch_moe_fp8(const MoeArgs& a, cudaStream_t s);
// The grouped linear on the persistent tile kernel (q8_gemm.cu); returns
// Q8_ERR_SHAPE for more experts than its tile map holds.
q8_status launch_grouped_fp8(const MoeArgs& a, cudaStream_t s);


}  // namespace q8
