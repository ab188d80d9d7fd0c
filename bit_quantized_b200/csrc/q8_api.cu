// The C ABI declared in include/q8.h: argument validation on the host, then
// kernel launches on the caller's stream.  Nothing here allocates device
// memory or synchronizes, except q8_get_device_status.
#include <cuda_runtime.h>

#include <atomic>
#include <cfloat>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "q8_internal.h"

namespace q8 {

// Per-device status word: 0, or the first device-side error (a bounded wait
// that ran out).  Kernels receive its address as an argument.
__device__ int g_device_status;

namespace {

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices];
int g_arch_ok[kMaxDevices];  // 0 unknown, 1 ok, 2 unsupported
std::mutex g_mu;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_bytes(q8_dtype d) {
    switch (d) {
        case Q8_S8: case Q8_U8: case Q8_E4M3: return 1;
        case Q8_F16: case Q8_BF16: return 2;
        case Q8_F32: case Q8_S32: return 4;
    }
    return 0;
}

bool float_input(q8_dtype d) { return d == Q8_F16 || d == Q8_BF16 || d == Q8_F32; }

bool ld_ok(int64_t ld, int64_t cols, q8_dtype d) {
    return ld >= cols && (ld * elem_bytes(d)) % 16 == 0;
}

constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;
constexpr int64_t kMaxKInt8 = 32768;

// Armed failure (q8_inject_failure): after `g_inject_skip` more validated
// calls, the next one returns `g_inject_code` before anything is enqueued.
std::atomic<int> g_inject_code{0};   // written under g_mu; read without it when unarmed
int g_inject_skip = 0;

q8_status device_ready() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return Q8_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_arch_ok[dev] == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
            cudaGetLastError();
            return Q8_ERR_CUDA;
        }
        g_arch_ok[dev] = (major == 10 && minor == 0) ? 1 : 2;
    }
    return g_arch_ok[dev] == 1 ? Q8_OK : Q8_ERR_UNSUPPORTED_ARCH;
}

// The last step of every launching entry point's checks: an armed injected
// failure, then the device.
q8_status check_device() {
    if (g_inject_code.load(std::memory_order_acquire) != 0) {
        std::lock_guard<std::mutex> lk(g_mu);
        const int code = g_inject_code.load(std::memory_order_relaxed);
        if (code != 0) {
            if (g_inject_skip > 0) {
                --g_inject_skip;
            } else {
                g_inject_code.store(0, std::memory_order_release);
                return static_cast<q8_status>(code);
            }
        }
    }
    return device_ready();
}

q8_status launch_status(cudaError_t e) {
    if (e == cudaSuccess) return Q8_OK;
    cudaGetLastError();
    return Q8_ERR_LAUNCH;
}

q8_status check_weight(const q8_weight* w) {
    if (!w) return Q8_ERR_NULL;
    if (w->n < 0 || w->k <= 0 || w->n > kMaxDim || w->k > kMaxDim || w->k % 32 != 0 ||
        w->n % 16 != 0 || w->ld < w->k)
        return Q8_ERR_SHAPE;
    if (w->n > 0 && (!w->codes || !w->scale)) return Q8_ERR_NULL;
    if (w->code_dtype != Q8_S8 && w->code_dtype != Q8_U8 && w->code_dtype != Q8_E4M3)
        return Q8_ERR_DTYPE;
    if (w->code_dtype == Q8_E4M3 && w->zero_point) return Q8_ERR_SCHEME;
    if (!aligned16(w->codes) || !aligned16(w->scale) ||
        (w->zero_point && !aligned16(w->zero_point)) || w->ld % 16 != 0)
        return Q8_ERR_ALIGN;
    return Q8_OK;
}

}  // namespace

int* device_status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_status_ptr[dev] = static_cast<int*>(p);
    }
    return g_status_ptr[dev];
}

}  // namespace q8

using namespace q8;

extern "C" {

int q8_version(void) { return Q8_VERSION; }

const char* q8_status_string(q8_status s) {
    switch (s) {
        case Q8_OK: return "ok";
        case Q8_ERR_NULL: return "a required pointer is NULL";
        case Q8_ERR_SHAPE: return "a size or leading dimension is out of range";
        case Q8_ERR_ALIGN: return "a pointer or leading dimension is not 16-byte aligned";
        case Q8_ERR_DTYPE: return "unsupported dtype or dtype combination";
        case Q8_ERR_SCHEME: return "unsupported scheme or scheme/code dtype mismatch";
        case Q8_ERR_UNSUPPORTED_ARCH: return "the current device is not compute capability 10.0 (sm_100a)";
        case Q8_ERR_LAUNCH: return "a kernel launch failed";
        case Q8_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait ran out";
        case Q8_ERR_WORKSPACE: return "workspace is NULL or too small";
        case Q8_ERR_CUDA: return "CUDA runtime error";
    }
    return "unknown status";
}

q8_status q8_device_check(void) { return device_ready(); }

q8_status q8_inject_failure(q8_status code, int32_t skip) {
    if (code < Q8_OK || code > Q8_ERR_CUDA) return Q8_ERR_SCHEME;
    if (skip < 0) return Q8_ERR_SHAPE;
    std::lock_guard<std::mutex> lk(g_mu);
    g_inject_skip = code == Q8_OK ? 0 : skip;
    g_inject_code.store(code, std::memory_order_release);
    return Q8_OK;
}

size_t q8_workspace_size(int op, int64_t m, int64_t n, int64_t k) {
    if (op != Q8_OP_LINEAR_INT8_MIXED || m < 0 || n < 0 || k < 0) return 0;
    // Beyond 2^31 - 1 no call is valid; the products below would also be
    // able to overflow int64 there.
    if (m > kMaxDim || n > kMaxDim || k > kMaxDim) return SIZE_MAX;
    auto up = [](int64_t v, int64_t a) { return (v + a - 1) / a * a; };
    const int64_t kp = up(k, 64);
    int64_t b = 0;
    b += up(k, 256);            // mask
    b += up(4 * k, 256);        // idx
    b += 256;                   // count
    b += up(m * k, 256);        // int8 codes
    b += up(4 * m, 256);        // scale
    b += up(4 * m, 256);        // rowsum
    b += up(2 * m * kp, 256);   // gathered outlier activations
    b += up(2 * n * kp, 256);   // gathered outlier weight columns
    return static_cast<size_t>(b);
}

q8_status q8_quantize_weight(const void* W, q8_dtype w_dtype, int64_t n, int64_t k, int64_t ldw,
                             q8_scheme scheme, q8_dtype code_dtype, void* codes, float* scale,
                             float* zero_point, q8_stream_t stream) {
    if (n < 0 || k <= 0 || n > kMaxDim || k > kMaxDim || k % 32 != 0) return Q8_ERR_SHAPE;
    if (!float_input(w_dtype)) return Q8_ERR_DTYPE;
    if (!(ldw >= k)) return Q8_ERR_SHAPE;
    switch (scheme) {
        case Q8_ASYM_INT8: if (code_dtype != Q8_S8 && code_dtype != Q8_U8) return Q8_ERR_SCHEME; break;
        case Q8_SYM_INT8: if (code_dtype != Q8_S8) return Q8_ERR_SCHEME; break;
        case Q8_FP8_E4M3: if (code_dtype != Q8_E4M3) return Q8_ERR_SCHEME; break;
        default: return Q8_ERR_SCHEME;
    }
    if (n == 0) return Q8_OK;   // empty call
    if (!W || !codes || !scale) return Q8_ERR_NULL;
    if (scheme == Q8_ASYM_INT8 && !zero_point) return Q8_ERR_NULL;
    if (!aligned16(W) || !aligned16(codes) || !ld_ok(ldw, k, w_dtype)) return Q8_ERR_ALIGN;
    q8_status st = check_device();
    if (st != Q8_OK) return st;
    RowQuantArgs a = {};
    a.src = W; a.src_dtype = w_dtype; a.rows = n; a.k = k; a.ld = ldw;
    a.op = scheme == Q8_ASYM_INT8 ? kOpWeightAsym : scheme == Q8_SYM_INT8 ? kOpWeightSym : kOpWeightFp8;
    a.codes_u8 = code_dtype == Q8_U8;
    a.codes = codes; a.scale = scale;
    a.zero_point = scheme == Q8_FP8_E4M3 ? nullptr : zero_point;
    return launch_status(launch_row_quant(a, reinterpret_cast<cudaStream_t>(stream)));
}

q8_status q8_dequantize_weight(const q8_weight* w, q8_dtype out_dtype, void* out,
                               q8_stream_t stream) {
    q8_status st = check_weight(w);
    if (st != Q8_OK) return st;
    if (!out) return Q8_ERR_NULL;
    if (!float_input(out_dtype)) return Q8_ERR_DTYPE;
    st = check_device();
    if (st != Q8_OK) return st;
    return launch_status(launch_dequant(*w, out_dtype, out, reinterpret_cast<cudaStream_t>(stream)));
}

q8_status q8_quantize_act(const void* X, q8_dtype x_dtype, int64_t m, int64_t k, int64_t ldx,
                          q8_scheme scheme, float clip_ub, void* codes, float* scale,
                          int32_t* rowsum, q8_stream_t stream) {
    if (m < 0 || k <= 0 || m > kMaxDim || k > kMaxDim || k % 32 != 0 || ldx < k) return Q8_ERR_SHAPE;
    if (!float_input(x_dtype)) return Q8_ERR_DTYPE;
    if (scheme != Q8_SYM_INT8 && scheme != Q8_FP8_E4M3) return Q8_ERR_SCHEME;
    if (m == 0) return Q8_OK;   // empty call: pointers may be NULL, nothing is launched
    if (!X || !codes || !scale) return Q8_ERR_NULL;
    if (!aligned16(X) || !aligned16(codes) || !ld_ok(ldx, k, x_dtype)) return Q8_ERR_ALIGN;
    q8_status st = check_device();
    if (st != Q8_OK) return st;
    RowQuantArgs a = {};
    a.src = X; a.src_dtype = x_dtype; a.rows = m; a.k = k; a.ld = ldx;
    a.op = scheme == Q8_SYM_INT8 ? kOpActInt8 : kOpActFp8;
    a.clip_ub = clip_ub;
    a.codes = codes; a.scale = scale;
    a.rowsum = scheme == Q8_SYM_INT8 ? rowsum : nullptr;
    return launch_status(launch_row_quant(a, reinterpret_cast<cudaStream_t>(stream)));
}

q8_status q8_quantize_act_static(const void* X, q8_dtype x_dtype, int64_t m, int64_t k, int64_t ldx,
                                 float static_scale, void* codes, float* scale, int32_t* rowsum,
                                 q8_stream_t stream) {
    if (m < 0 || k <= 0 || m > kMaxDim || k > kMaxDim || k % 32 != 0 || ldx < k) return Q8_ERR_SHAPE;
    if (!float_input(x_dtype)) return Q8_ERR_DTYPE;
    if (!(static_scale > 0.0f) || !(static_scale <= FLT_MAX)) return Q8_ERR_SCHEME;
    if (m == 0) return Q8_OK;   // empty call
    if (!X || !codes || !scale) return Q8_ERR_NULL;
    if (!aligned16(X) || !aligned16(codes) || !ld_ok(ldx, k, x_dtype)) return Q8_ERR_ALIGN;
    q8_status st = check_device();
    if (st != Q8_OK) return st;
    RowQuantArgs a = {};
    a.src = X; a.src_dtype = x_dtype; a.rows = m; a.k = k; a.ld = ldx;
    a.op = kOpActInt8Static;
    a.static_scale = static_scale;
    a.codes = codes; a.scale = scale; a.rowsum = rowsum;
    return launch_status(launch_row_quant(a, reinterpret_cast<cudaStream_t>(stream)));
}

q8_status q8_quantize_act_smooth(const void* X, q8_dtype x_dtype, int64_t m, int64_t k, int64_t ldx,
                                 const float* mult, void* codes, float* scale, int32_t* rowsum,
                                 q8_stream_t stream) {
    if (m < 0 || k <= 0 || m > kMaxDim || k > kMaxDim || k % 32 != 0 || ldx < k) return Q8_ERR_SHAPE;
    if (!float_input(x_dtype)) return Q8_ERR_DTYPE;
    if (m == 0) return Q8_OK;   // empty call
    if (!X || !codes || !scale || !mult) return Q8_ERR_NULL;
    if (!aligned16(X) || !aligned16(codes) || !aligned16(mult) || !ld_ok(ldx, k, x_dtype))
        return Q8_ERR_ALIGN;
    q8_status st = check_device();
    if (st != Q8_OK) return st;
    RowQuantArgs a = {};
    a.src = X; a.src_dtype = x_dtype; a.rows = m; a.k = k; a.ld = ldx;
    a.op = kOpActInt8Smooth;
    a.mult = mult;
    a.codes = codes; a.scale = scale; a.rowsum = rowsum;
    return launch_status(launch_row_quant(a, reinterpret_cast<cudaStream_t>(stream)));
}

static q8_status validate_outlier_act(const void* X, q8_dtype x_dtype, int64_t m, int64_t k,
                                      int64_t ldx, void* codes, float* scale, int32_t* rowsum,
                                      uint8_t* mask, int32_t* idx, int32_t* count,
                                      void* x_outlier, int64_t ldo) {
    if (!mask || !idx || !count) return Q8_ERR_NULL;
    if (m < 0 || k <= 0 || m > kMaxDim || k > kMaxKInt8 || k % 32 != 0 || ldx < k) return Q8_ERR_SHAPE;
    if (m > 0 && (!X || !codes || !scale || !rowsum)) return Q8_ERR_NULL;
    if (x_outlier && (ldo < (k + 63) / 64 * 64)) return Q8_ERR_SHAPE;
    if (x_dtype != Q8_F16) return Q8_ERR_DTYPE;
    if (!aligned16(X) || !aligned16(codes) || !ld_ok(ldx, k, x_dtype) || !aligned16(mask))
        return Q8_ERR_ALIGN;
    if (x_outlier && (!aligned16(x_outlier) || ldo % 8 != 0)) return Q8_ERR_ALIGN;
    return Q8_OK;
}

// Two launches: the column absmax pass writes the outlier mask (every token
// must be seen before any row is coded), then the row pass ranks the outlier
// columns, codes the regular stream and gathers the fp16 outlier columns of X
// and, when `w` is given, of the weight.
static q8_status run_outlier_act(const void* X, int64_t m, int64_t k, int64_t ldx, float threshold,
                                 void* codes, float* scale, int32_t* rowsum, uint8_t* mask,
                                 int32_t* idx, int32_t* count, void* x_outlier, int64_t ldo,
                                 const q8_weight* w, const void* W16, void* w_outlier,
                                 cudaStream_t s) {
    cudaError_t e = launch_outlier_columns(X, Q8_F16, m, k, ldx, threshold, mask, s);
    if (e != cudaSuccess) return launch_status(e);
    if (m == 0) return launch_status(cudaMemsetAsync(count, 0, sizeof(int32_t), s));   // no rows: no outliers
    RowQuantArgs a = {};
    a.src = X; a.src_dtype = Q8_F16; a.rows = m; a.k = k; a.ld = ldx;
    a.op = kOpActInt8;
    a.skip = mask;
    a.codes = codes; a.scale = scale; a.rowsum = rowsum;
    a.outlier_idx = idx; a.outlier_count = count;
    a.x_outlier = static_cast<__half*>(x_outlier);
    a.ldo = ldo;
    if (w != nullptr) {
        a.w_rows = w->n;
        a.w_codes = w->codes;
        a.w_codes_u8 = w->code_dtype == Q8_U8;
        a.w_ld = W16 ? k : w->ld;
        a.w_scale = w->scale;
        a.w_zero = w->zero_point;
        a.w16 = static_cast<const __half*>(W16);
        a.w_outlier = static_cast<__half*>(w_outlier);
    }
    return launch_status(launch_row_quant(a, s));
}

q8_status q8_outlier_quantize_act(const void* X, q8_dtype x_dtype, int64_t m, int64_t k,
                                  int64_t ldx, float threshold, void* codes, float* scale,
                                  int32_t* rowsum, uint8_t* mask, int32_t* idx, int32_t* count,
                                  void* x_outlier, int64_t ldo, q8_stream_t stream) {
    q8_status st = validate_outlier_act(X, x_dtype, m, k, ldx, codes, scale, rowsum, mask, idx,
                                        count, x_outlier, ldo);
    if (st != Q8_OK) return st;
    st = check_device();
    if (st != Q8_OK) return st;
    return run_outlier_act(X, m, k, ldx, threshold, codes, scale, rowsum, mask, idx, count,
                           x_outlier, ldo, nullptr, nullptr, nullptr,
                           reinterpret_cast<cudaStream_t>(stream));
}

q8_status q8_linear_w8a8(const q8_act* x, const q8_weight* w, const float* bias, void* Y,
                         int64_t ldy, void* acc_debug, void* workspace, size_t ws_bytes,
                         q8_stream_t stream) {
    (void)workspace;
    (void)ws_bytes;
    q8_status st = check_weight(w);
    if (st != Q8_OK) return st;
    if (!x) return Q8_ERR_NULL;
    if (x->m < 0 || x->m > kMaxDim || x->k != w->k || x->ld < x->k || ldy < w->n) return Q8_ERR_SHAPE;
    const bool fp8 = x->code_dtype == Q8_E4M3;
    if (fp8 != (w->code_dtype == Q8_E4M3) || (x->code_dtype != Q8_S8 && !fp8)) return Q8_ERR_DTYPE;
    if (!fp8 && w->k > kMaxKInt8) return Q8_ERR_SHAPE;
    if (x->m == 0 || w->n == 0) return Q8_OK;   // empty call
    if (!x->codes || !x->scale || !Y) return Q8_ERR_NULL;
    if (!fp8 && w->zero_point && !x->rowsum) return Q8_ERR_NULL;
    if (!aligned16(x->codes) || !aligned16(x->scale) || x->ld % 16 != 0 || !aligned16(Y) ||
        ldy % 8 != 0 || (bias && !aligned16(bias)) || (acc_debug && !aligned16(acc_debug)))
        return Q8_ERR_ALIGN;
    st = check_device();
    if (st != Q8_OK) return st;
    LinearArgs a = {};
    a.m = x->m; a.n = w->n; a.k = w->k;
    a.a_codes = x->codes; a.lda = x->ld;
    a.b_codes = w->codes; a.ldb = w->ld;
    a.kind = fp8 ? 2 : (w->code_dtype == Q8_U8 ? 1 : 0);
    a.sx = x->scale; a.rowsum = fp8 ? nullptr : x->rowsum;
    a.sw = w->scale; a.zw = fp8 ? nullptr : w->zero_point;
    a.bias = bias;
    a.y = static_cast<__nv_bfloat16*>(Y); a.ldy = ldy;
    a.acc_debug = acc_debug;
    return launch_linear(a, reinterpret_cast<cudaStream_t>(stream));
}

q8_status q8_linear_w8a8_requant(const q8_act* x, const q8_weight* w, const float* bias,
                                 float out_scale, void* Yq, int64_t ldy, void* acc_debug,
                                 q8_stream_t stream) {
    q8_status st = check_weight(w);
    if (st != Q8_OK) return st;
    if (!x) return Q8_ERR_NULL;
    if (x->m < 0 || x->m > kMaxDim || x->k != w->k || x->ld < x->k || ldy < w->n) return Q8_ERR_SHAPE;
    if (x->code_dtype != Q8_S8 || w->code_dtype == Q8_E4M3) return Q8_ERR_DTYPE;
    if (w->k > kMaxKInt8) return Q8_ERR_SHAPE;
    if (!(out_scale > 0.0f) || !(out_scale <= FLT_MAX)) return Q8_ERR_SCHEME;
    if (x->m == 0 || w->n == 0) return Q8_OK;   // empty call
    if (!x->codes || !x->scale || !Yq) return Q8_ERR_NULL;
    if (w->zero_point && !x->rowsum) return Q8_ERR_NULL;
    if (!aligned16(x->codes) || !aligned16(x->scale) || x->ld % 16 != 0 || !aligned16(Yq) ||
        ldy % 16 != 0 || (bias && !aligned16(bias)) || (acc_debug && !aligned16(acc_debug)))
        return Q8_ERR_ALIGN;
    st = check_device();
    if (st != Q8_OK) return st;
    LinearArgs a = {};
    a.m = x->m; a.n = w->n; a.k = w->k;
    a.a_codes = x->codes; a.lda = x->ld;
    a.b_codes = w->codes; a.ldb = w->ld;
    a.kind = w->code_dtype == Q8_U8 ? 1 : 0;
    a.sx = x->scale; a.rowsum = x->rowsum;
    a.sw = w->scale; a.zw = w->zero_point;
    a.bias = bias;
    a.yq = static_cast<int8_t*>(Yq); a.out_scale = out_scale; a.ldy = ldy;
    a.acc_debug = acc_debug;
    return launch_linear(a, reinterpret_cast<cudaStream_t>(stream));
}

q8_status q8_linear_w8a8_dynamic(const void* X, q8_dtype x_dtype, int64_t m, int64_t k,
                                 int64_t ldx, q8_scheme act_scheme, float clip_ub,
                                 const q8_weight* w, const float* bias, void* Y, int64_t ldy,
                                 void* act_codes, float* act_scale, int32_t* act_rowsum,
                                 void* acc_debug, q8_stream_t stream) {
    q8_status st = check_weight(w);
    if (st != Q8_OK) return st;
    if (m < 0 || m > kMaxDim || k != w->k || ldx < k || ldy < w->n) return Q8_ERR_SHAPE;
    if (!float_input(x_dtype)) return Q8_ERR_DTYPE;
    const bool fp8 = act_scheme == Q8_FP8_E4M3;
    if (act_scheme != Q8_SYM_INT8 && !fp8) return Q8_ERR_SCHEME;
    if (fp8 != (w->code_dtype == Q8_E4M3)) return Q8_ERR_DTYPE;
    if (!fp8 && w->k > kMaxKInt8) return Q8_ERR_SHAPE;
    if (m == 0 || w->n == 0) return Q8_OK;   // empty call
    if (!X || !Y || !act_codes || !act_scale || (!fp8 && !act_rowsum)) return Q8_ERR_NULL;
    if (!aligned16(X) || !ld_ok(ldx, k, x_dtype) || !aligned16(Y) || ldy % 8 != 0 ||
        !aligned16(act_codes) || !aligned16(act_scale) || (bias && !aligned16(bias)) ||
        (acc_debug && !aligned16(acc_debug)))
        return Q8_ERR_ALIGN;
    st = check_device();
    if (st != Q8_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    LinearArgs a = {};
    a.m = m; a.n = w->n; a.k = k;
    a.a_codes = act_codes; a.lda = k;
    a.b_codes = w->codes; a.ldb = w->ld;
    a.kind = fp8 ? 2 : (w->code_dtype == Q8_U8 ? 1 : 0);
    a.sx = act_scale; a.rowsum = fp8 ? nullptr : act_rowsum;
    a.sw = w->scale; a.zw = fp8 ? nullptr : w->zero_point;
    a.bias = bias;
    a.y = static_cast<__nv_bfloat16*>(Y); a.ldy = ldy;
    a.acc_debug = acc_debug;
    // The quantizer lets the GEMM start early (programmatic dependent launch):
    // the GEMM's prologue and weight loads overlap the quantization.
    RowQuantArgs r = {};
    r.src = X; r.src_dtype = x_dtype; r.rows = m; r.k = k; r.ld = ldx;
    r.op = fp8 ? kOpActFp8 : kOpActInt8;
    r.clip_ub = clip_ub;
    r.codes = act_codes; r.scale = act_scale;
    r.rowsum = fp8 ? nullptr : act_rowsum;
    st = launch_status(launch_row_quant(r, s));
    if (st != Q8_OK) return st;
    return launch_linear(a, s);
}

q8_status q8_linear_int8_mixed(const void* X, q8_dtype x_dtype, int64_t m, int64_t k, int64_t ldx,
                               const q8_weight* w, const void* W16, float threshold,
                               const float* bias, void* Y, int64_t ldy, uint8_t* outlier_mask,
                               int32_t* outlier_count, int32_t* acc_debug, float* y16_debug,
                               void* workspace, size_t ws_bytes, q8_stream_t stream) {
    q8_status st = check_weight(w);
    if (st != Q8_OK) return st;
    if (w->code_dtype == Q8_E4M3) return Q8_ERR_DTYPE;
    if (x_dtype != Q8_F16) return Q8_ERR_DTYPE;
    if (m < 0 || m > kMaxDim || k != w->k || k > kMaxKInt8 || ldx < k || ldy < w->n) return Q8_ERR_SHAPE;
    if (m == 0 || w->n == 0) return Q8_OK;   // empty call
    if (!X || !Y) return Q8_ERR_NULL;
    if (!aligned16(X) || !ld_ok(ldx, k, x_dtype) || !aligned16(Y) || ldy % 8 != 0 ||
        (W16 && !aligned16(W16)) || (bias && !aligned16(bias)) ||
        (acc_debug && !aligned16(acc_debug)) || (y16_debug && !aligned16(y16_debug)))
        return Q8_ERR_ALIGN;
    const size_t need = q8_workspace_size(Q8_OP_LINEAR_INT8_MIXED, m, w->n, k);
    if (!workspace || ws_bytes < need) return Q8_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return Q8_ERR_ALIGN;
    st = check_device();
    if (st != Q8_OK) return st;

    auto up = [](int64_t v, int64_t a) { return (v + a - 1) / a * a; };
    const int64_t kp = up(k, 64);
    uint8_t* p = static_cast<uint8_t*>(workspace);
    uint8_t* mask = p;              p += up(k, 256);
    int32_t* idx = reinterpret_cast<int32_t*>(p); p += up(4 * k, 256);
    int32_t* count = reinterpret_cast<int32_t*>(p); p += 256;
    int8_t* codes = reinterpret_cast<int8_t*>(p); p += up(m * k, 256);
    float* sx = reinterpret_cast<float*>(p); p += up(4 * m, 256);
    int32_t* rowsum = reinterpret_cast<int32_t*>(p); p += up(4 * m, 256);
    __half* xo = reinterpret_cast<__half*>(p); p += up(2 * m * kp, 256);
    __half* wo = reinterpret_cast<__half*>(p);

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    st = run_outlier_act(X, m, k, ldx, threshold, codes, sx, rowsum, mask, idx, count, xo, kp, w,
                         W16, wo, s);
    if (st != Q8_OK) return st;
    LinearArgs a = {};
    a.m = m; a.n = w->n; a.k = k;
    a.a_codes = codes; a.lda = k;
    a.b_codes = w->codes; a.ldb = w->ld;
    a.kind = w->code_dtype == Q8_U8 ? 1 : 0;
    a.sx = sx; a.rowsum = rowsum;
    a.sw = w->scale; a.zw = w->zero_point;
    a.bias = bias;
    a.y = static_cast<__nv_bfloat16*>(Y); a.ldy = ldy;
    a.acc_debug = acc_debug;
    a.xo = xo; a.ldxo = kp;
    a.wo = wo; a.ldwo = kp;
    a.outlier_count = count;
    a.k16_cap = kp;
    a.y16_debug = y16_debug;
    st = launch_linear(a, s);
    if (st != Q8_OK) return st;
    if (outlier_mask &&
        cudaMemcpyAsync(outlier_mask, mask, static_cast<size_t>(k), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return launch_status(cudaErrorUnknown);
    if (outlier_count &&
        cudaMemcpyAsync(outlier_count, count, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return launch_status(cudaErrorUnknown);
    return Q8_OK;
}

q8_status q8_quantize_weight_g4(const void* W, q8_dtype w_dtype, int64_t n, int64_t k,
                                int64_t ldw, int32_t group, void* codes, int64_t ldc,
                                float* scale, q8_stream_t stream) {
    if (w_dtype != Q8_F16 && w_dtype != Q8_BF16) return Q8_ERR_DTYPE;
    if (group != 32 && group != 64 && group != 128) return Q8_ERR_SCHEME;
    if (n < 0 || k <= 0 || n > kMaxDim || k > kMaxDim || k % 32 != 0 || k % group != 0 ||
        n % 16 != 0 || ldw < k || ldc < k / 2)
        return Q8_ERR_SHAPE;
    if (n == 0) return Q8_OK;
    if (!W || !codes || !scale) return Q8_ERR_NULL;
    if (!aligned16(W) || !ld_ok(ldw, k, w_dtype) || !aligned16(codes) || ldc % 16 != 0 ||
        !aligned16(scale))
        return Q8_ERR_ALIGN;
    q8_status st = check_device();
    if (st != Q8_OK) return st;
    return launch_status(launch_group_quant(W, w_dtype, n, k, ldw, group,
                                            static_cast<uint8_t*>(codes), ldc, scale,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

q8_status q8_quantize_weight_q4k(const void* W, q8_dtype w_dtype, int64_t n, int64_t k,
                                 int64_t ldw, void* codes, int64_t ldc, float* scale,
                                 uint8_t* sub_codes, float* super_scale, q8_stream_t stream) {
    if (w_dtype != Q8_F16 && w_dtype != Q8_BF16) return Q8_ERR_DTYPE;
    if (n < 0 || k <= 0 || n > kMaxDim || k > kMaxDim || k % 256 != 0 || n % 16 != 0 || ldw < k ||
        ldc < k / 2)
        return Q8_ERR_SHAPE;
    if (n == 0) return Q8_OK;
    if (!W || !codes || !scale || !sub_codes || !super_scale) return Q8_ERR_NULL;
    if (!aligned16(W) || !ld_ok(ldw, k, w_dtype) || !aligned16(codes) || ldc % 16 != 0 ||
        !aligned16(scale) || !aligned16(sub_codes) || !aligned16(super_scale))
        return Q8_ERR_ALIGN;
    q8_status st = check_device();
    if (st != Q8_OK) return st;
    return launch_status(launch_q4k_quant(W, w_dtype, n, k, ldw, static_cast<uint8_t*>(codes), ldc,
                                          scale, sub_codes, super_scale,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

q8_status q8_expand_q4k_scales(const uint8_t* sub_codes, const float* super_scale, int64_t n,
                               int64_t k, float* scale, q8_stream_t stream) {
    if (n < 0 || k <= 0 || n > kMaxDim || k > kMaxDim || k % 256 != 0 || n % 16 != 0)
        return Q8_ERR_SHAPE;
    if (n == 0) return Q8_OK;
    if (!sub_codes || !super_scale || !scale) return Q8_ERR_NULL;
    if (!aligned16(sub_codes) || !aligned16(super_scale) || !aligned16(scale)) return Q8_ERR_ALIGN;
    q8_status st = check_device();
    if (st != Q8_OK) return st;
    return launch_status(launch_q4k_expand(sub_codes, super_scale, n, k, scale,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

q8_status q8_linear_w4a16(const void* X, q8_dtype x_dtype, int64_t m, int64_t k, int64_t ldx,
                          const q8_weight_g4* w, const float* bias, void* Y, int64_t ldy,
                          q8_stream_t stream) {
    if (!w) return Q8_ERR_NULL;
    if (x_dtype != Q8_F16 && x_dtype != Q8_BF16) return Q8_ERR_DTYPE;
    if (w->group != 32 && w->group != 64 && w->group != 128) return Q8_ERR_SCHEME;
    if (w->n < 0 || w->k <= 0 || w->n > kMaxDim || w->k > kMaxDim || w->k % 32 != 0 ||
        w->k % w->group != 0 || w->n % 16 != 0 || w->ld < w->k / 2)
        return Q8_ERR_SHAPE;
    // token tiles of up to 256 along the grid's z dimension (at most 65535)
    if (m < 0 || m > int64_t(65535) * 256 || k != w->k || ldx < k || ldy < w->n) return Q8_ERR_SHAPE;
    if (m == 0 || w->n == 0) return Q8_OK;   // empty call
    if (!X || !Y || !w->codes || !w->scale) return Q8_ERR_NULL;
    if (!aligned16(X) || !ld_ok(ldx, k, x_dtype) || !aligned16(Y) || ldy % 8 != 0 ||
        !aligned16(w->codes) || w->ld % 16 != 0 || !aligned16(w->scale) ||
        (bias && !aligned16(bias)))
        return Q8_ERR_ALIGN;
    q8_status st = check_device();
    if (st != Q8_OK) return st;
    W4Args a = {};
    a.x = X; a.x_bf16 = x_dtype == Q8_BF16;
    a.m = m; a.k = k; a.ldx = ldx;
    a.codes = w->codes; a.ldc = w->ld;
    a.scale = w->scale;
    a.n = w->n;
    a.group = w->group;
    a.bias = bias;
    a.y = static_cast<__nv_bfloat16*>(Y); a.ldy = ldy;
    return launch_w4a16(a, reinterpret_cast<cudaStream_t>(stream));
}

q8_status q8_linear_fp8_grouped(const q8_act* x, const q8_weight* w, int64_t num_experts,
                                const int32_t* offsets, const float* bias, void* Y, int64_t ldy,
                                q8_stream_t stream) {
    if (!x || !w) return Q8_ERR_NULL;
    q8_status st = check_weight(w);
    if (st != Q8_OK) return st;
    if (x->code_dtype != Q8_E4M3 || w->code_dtype != Q8_E4M3) return Q8_ERR_DTYPE;
    if (num_experts < 1 || num_experts > 4096 || w->n % num_experts != 0) return Q8_ERR_SHAPE;
    const int64_t n = w->n / num_experts;
    if (n % 16 != 0 || x->m < 0 || x->m > kMaxDim || x->k != w->k || x->ld < x->k || ldy < n ||
        (x->m + 127) / 128 + num_experts > 65535)
        return Q8_ERR_SHAPE;
    if (x->m == 0 || n == 0) return Q8_OK;   // empty call
    if (!x->codes || !x->scale || !offsets || !Y) return Q8_ERR_NULL;
    if (!aligned16(x->codes) || x->ld % 16 != 0 || !aligned16(x->scale) || !aligned16(Y) ||
        ldy % 8 != 0 || (bias && !aligned16(bias)) || (reinterpret_cast<uintptr_t>(offsets) & 3u))
        return Q8_ERR_ALIGN;
    st = check_device();
    if (st != Q8_OK) return st;
    MoeArgs a = {};
    a.m = x->m; a.k = x->k;
    a.x_codes = x->codes; a.ldx = x->ld; a.sx = x->scale;
    a.experts = num_experts; a.n = n;
    a.w_codes = w->codes; a.ldw = w->ld; a.sw = w->scale;
    a.offsets = offsets;
    a.bias = bias;
    a.y = static_cast<__nv_bfloat16*>(Y); a.ldy = ldy;
    return launch_moe_fp8(a, reinterpret_cast<cudaStream_t>(stream));
}

q8_status q8_get_device_status(int32_t* out, q8_stream_t stream) {
    if (!out) return Q8_ERR_NULL;
    q8_status st = device_ready();
    if (st != Q8_OK) return st;
    int* p = device_status_ptr();
    if (!p) return Q8_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int v = 0;
    if (cudaMemcpyAsync(&v, p, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return Q8_ERR_CUDA;
    }
    *out = v;
    return Q8_OK;
}

q8_status q8_clear_device_status(q8_stream_t stream) {
    q8_status st = device_ready();
    if (st != Q8_OK) return st;
    int* p = device_status_ptr();
    if (!p) return Q8_ERR_CUDA;
    if (cudaMemsetAsync(p, 0, sizeof(int), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return Q8_ERR_CUDA;
    }
    return Q8_OK;
}

}  // extern "C"
