// Quantize kernels: per-row (token or output channel) reductions followed by
// the elementwise quantization of the same row, plus the LLM.int8 outlier
// column pass.  All of them are bound by HBM bandwidth: each reads its input
// once with 16-byte vector loads, keeps the row in registers between the
// reduction and the quantization, and writes packed codes.
//
// Arithmetic is the pages' closed forms in IEEE fp32 with explicit
// round-to-nearest intrinsics, so the codes are bit-identical to a scalar
// evaluation of the same formulas:
//   symmetric   S = max(absmax / qmax, 1e-8), q = clamp(rne(x / S), -qmax, qmax)
//               ("大模型量化" (Xilyfe), symmetric section: s = (2^(b-1) - 1) / alpha)
//   asymmetric  S = max((max - min) / 255, 1e-8), Z = clamp(rne(-min / S) - 128),
//               q = clamp(rne(w / S) + Z, -128, 127)
//               (same page, asymmetric section; 8-Bit LLM Quantization with
//               Lightning Fabric, sections 2.1 and 2.3)
//   FP8         S = max(min(absmax, ub) / 448, 1e-8), q = e4m3_rne_satfinite(x / S)
//               (Transformers FP8 (W8A8) / FBGEMM page, sections 5.1, 5.2 and 6)
//   static      S given (calibrated offline), q = clamp(rne(x / S), -127, 127)
//               ("大模型量化" (Xilyfe), the paragraph on static quantization)
//   smoothed    xs = x * m_col (m = 1 / smoothing factor), then symmetric on xs
//               (same page, algorithm list, SmoothQuant)
// Every x / S above is the IEEE fp32 quotient; the kernels reach its rounding
// without a division per element (see "Codes of one 16-byte vector" below).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>
#include <type_traits>

#include "q8_device.cuh"
#include "q8_internal.h"
#include "q8_qmath.cuh"

namespace q8 {
namespace {

using qm::kEps;
using qm::kMagic;
constexpr int kBlock = 256;
constexpr int kMaxVec = 16;   // 16-byte vectors a thread keeps in registers

template <typename T> struct VecOf;
template <> struct VecOf<__half> { static constexpr int N = 8; };
template <> struct VecOf<__nv_bfloat16> { static constexpr int N = 8; };
template <> struct VecOf<float> { static constexpr int N = 4; };

// Read-only streaming load (not volatile, so the compiler can issue all of a
// thread's loads before the first use and keep them in flight together).
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 u;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w)
        : "l"(p));
    return u;
}

template <typename T>
__device__ __forceinline__ void unpack_vec(const uint4 u, float (&v)[VecOf<T>::N]) {
    if constexpr (VecOf<T>::N == 4) {
        v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y);
        v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
    } else {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if constexpr (sizeof(T) == 2 && std::is_same<T, __half>::value) {
                const __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
                const float2 f = __half22float2(h);
                v[2 * i] = f.x; v[2 * i + 1] = f.y;
            } else {
                const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
                const float2 f = __bfloat1622float2(h);
                v[2 * i] = f.x; v[2 * i + 1] = f.y;
            }
        }
    }
}

template <typename T>
__device__ __forceinline__ void load_vec(const T* p, float (&v)[VecOf<T>::N]) {
    unpack_vec<T>(ld_stream16(p), v);
}

struct RowStats {
    float amax, lo, hi;
};

// Barrier over the TPR threads of one row group (named barrier 1 + group;
// the whole block when one group fills it).
template <int TPR>
__device__ __forceinline__ void group_sync() {
    if constexpr (TPR >= kBlock) {
        __syncthreads();
    } else {
        asm volatile("bar.sync %0, %1;" ::"r"(1 + static_cast<int>(threadIdx.x) / TPR), "n"(TPR) : "memory");
    }
}

// Reduction of per-thread stats over the TPR threads that share a row.
template <int TPR, bool MINMAX>
__device__ __forceinline__ RowStats group_reduce(RowStats s, float* red) {
#pragma unroll
    for (int o = (TPR < 32 ? TPR : 32) / 2; o > 0; o >>= 1) {
        if constexpr (MINMAX) {
            s.lo = fminf(s.lo, __shfl_xor_sync(0xffffffffu, s.lo, o));
            s.hi = fmaxf(s.hi, __shfl_xor_sync(0xffffffffu, s.hi, o));
        } else {
            s.amax = fmaxf(s.amax, __shfl_xor_sync(0xffffffffu, s.amax, o));
        }
    }
    if constexpr (TPR > 32) {
        constexpr int W = TPR / 32;
        const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
        if (lane == 0) {
            red[3 * warp] = s.amax; red[3 * warp + 1] = s.lo; red[3 * warp + 2] = s.hi;
        }
        group_sync<TPR>();
        const int base = (warp / W) * W;
        RowStats r{0.f, FLT_MAX, -FLT_MAX};
#pragma unroll
        for (int i = 0; i < W; ++i) {
            r.amax = fmaxf(r.amax, red[3 * (base + i)]);
            r.lo = fminf(r.lo, red[3 * (base + i) + 1]);
            r.hi = fmaxf(r.hi, red[3 * (base + i) + 2]);
        }
        group_sync<TPR>();
        return r;
    }
    return s;
}

template <int TPR>
__device__ __forceinline__ int group_sum(int v, int* red) {
#pragma unroll
    for (int o = (TPR < 32 ? TPR : 32) / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if constexpr (TPR > 32) {
        constexpr int W = TPR / 32;
        const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
        if (lane == 0) red[warp] = v;
        group_sync<TPR>();
        const int base = (warp / W) * W;
        int r = 0;
#pragma unroll
        for (int i = 0; i < W; ++i) r += red[base + i];
        group_sync<TPR>();
        return r;
    }
    return v;
}

__device__ __forceinline__ float clampf(float v, float lo, float hi) {
    return fminf(fmaxf(v, lo), hi);
}


// Codes of one 16-byte vector (V elements) without a division per element.
//
// The target is a rounding of the IEEE quotient fl32(x / S): rne for integer
// codes, E4M3 (half to even, saturating) for FP8.  Each row gets R = RN(1/S)
// and the next 24 bits of 1/S, and every element's quotient is formed exactly
// from them with a multiply, an FMA and one FMA correction (qm::quotient2:
// Markstein's correction step from a faithful first quotient).  No element
// needs a division, and there is no special case for quotients that fall on a
// rounding boundary (with 16-bit inputs, x / S falls exactly on one about 2
// times in 1000: 127 x / absmax is a ratio of two short significands).
//   Integer codes: t = RN(q + 1.5 * 2^23) lies in [2^23, 2^24), where floats
//   are the integers, so t is q rounded half to even and the low byte of t's
//   bits is the code's two's-complement byte.  The code range [-127, 127]
//   (static), or [-128, 127] after adding Z (asymmetric), is applied to q
//   before the rounding: its bounds are integers, so clamping first and
//   rounding second give the same code.  Z and the unsigned-storage bias are
//   added after the rounding (added before it, an odd Z would move the ties).
//   Dynamic symmetric rows need no clamp: |x| <= absmax makes |q| <= 127
//   (1 + 2^-23).
//   E4M3 codes: the hardware conversion of q (round to nearest even,
//   saturating to 448).
// Rows whose quotients could reach 2^99 (a static or clipped scale far below
// the row's values, asymmetric rows far from zero) or whose scale is below
// 2^-90 are coded with an IEEE division per element instead.

// Internal op for the LLM.int8 regular stream: int8 activations with the
// outlier columns (mask bytes of 1) left out of the absmax and coded as 0.
constexpr int kOpActInt8Skip = 5;

__host__ __device__ constexpr bool is_fp8_op(int op) { return op == kOpActFp8 || op == kOpWeightFp8; }

__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
    return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

__device__ __forceinline__ float2 splat2(float a) { return make_float2(a, a); }

// Per-row constants.
struct RowConsts {
    float S, Z, bias;
    float R, Rlo;     // RN(1/S) and the next bits of 1/S
    float qlo, qhi;   // integer codes: bounds of q before the rounding
    float post;       // integer codes: Z + bias, added after the rounding
    bool direct;      // code the row with a division per element
};

template <int OP>
__device__ __forceinline__ RowConsts row_consts(float amax, float lo, float hi, float clip_ub, float bias,
                                                float static_scale) {
    RowConsts c;
    c.Z = 0.f;
    c.bias = bias;
    float vmax = amax;   // largest |x| of the row
    if constexpr (OP == kOpActInt8Static) {
        c.S = static_scale;   // calibrated, > 0 (checked by the caller)
    } else if constexpr (OP == kOpActInt8 || OP == kOpActInt8Skip || OP == kOpActInt8Smooth ||
                         OP == kOpWeightSym) {
        c.S = __fdiv_rn(amax, 127.0f);
    } else if constexpr (is_fp8_op(OP)) {
        if (OP == kOpActFp8 && clip_ub > 0.f) amax = fminf(amax, clip_ub);
        c.S = __fdiv_rn(amax, 448.0f);
    } else {
        c.S = __fdiv_rn(__fsub_rn(hi, lo), 255.0f);
        vmax = fmaxf(fabsf(lo), fabsf(hi));
    }
    if (OP != kOpActInt8Static && !(c.S >= kEps)) c.S = kEps;
    c.R = __frcp_rn(c.S);
    c.Rlo = qm::reciprocal_low(c.S, c.R);
    c.qlo = -127.0f;
    c.qhi = 127.0f;
    c.post = 0.f;
    if constexpr (OP == kOpWeightAsym) {
        c.Z = clampf(__fsub_rn(rintf(__fdiv_rn(-lo, c.S)), 128.0f), -128.0f, 127.0f);
        c.qlo = -128.0f - c.Z;   // integers: exact
        c.qhi = 127.0f - c.Z;
        c.post = c.Z + bias;
    }
    // NaN-safe: a NaN or infinite product also takes the division.
    c.direct = !(vmax * c.R < qm::kQuotientMax) || !(c.S >= qm::kScaleMin);
    return c;
}

// Multipliers of a vector's columns (activation smoothing), from L1.
template <int V>
__device__ __forceinline__ void load_mult(const float* mult, int64_t j, float (&m)[V]) {
    const float4* p = reinterpret_cast<const float4*>(mult + j * V);
    const float4 a = __ldg(p);
    m[0] = a.x; m[1] = a.y; m[2] = a.z; m[3] = a.w;
    if constexpr (V == 8) {
        const float4 b = __ldg(p + 1);
        m[4] = b.x; m[5] = b.y; m[6] = b.z; m[7] = b.w;
    }
}

// Unpacked values of a vector; smoothed activations are fl32(x * m) per column.
template <typename T, int OP>
__device__ __forceinline__ void values_of(const uint4 u, const float* mv, float (&v)[VecOf<T>::N]) {
    unpack_vec<T>(u, v);
    if constexpr (OP == kOpActInt8Smooth) {
#pragma unroll
        for (int e = 0; e < VecOf<T>::N; ++e) v[e] = __fmul_rn(v[e], mv[e]);
    }
}

// Codes of one vector, packed in element order (element 4w + b in byte b of
// word w).  keep clears the bytes of left-out columns (all ones otherwise).
// DIRECT divides (rows outside the quotient's exact domain).
template <typename T, int OP, bool DIRECT>
__device__ __forceinline__ uint2 code_vec(const uint4 u, const RowConsts& c, const uint2 keep,
                                          const float* mv = nullptr) {
    constexpr int V = VecOf<T>::N;
    float v[V];
    values_of<T, OP>(u, mv, v);
    float2 q[V / 2];
    if constexpr (DIRECT) {
#pragma unroll
        for (int e = 0; e < V / 2; ++e) q[e] = make_float2(__fdiv_rn(v[2 * e], c.S), __fdiv_rn(v[2 * e + 1], c.S));
    } else {
        const float2 nS = splat2(-c.S), R = splat2(c.R), Rlo = splat2(c.Rlo);
#pragma unroll
        for (int e = 0; e < V / 2; ++e)
            q[e] = qm::quotient2(make_float2(v[2 * e], v[2 * e + 1]), nS, R, Rlo);
    }
    uint32_t words[2] = {0u, 0u};
    if constexpr (is_fp8_op(OP)) {
        // The quotient of -0 comes out as +0; every other quotient has x's
        // sign.  E4M3 keeps the sign of zero, so each code byte takes the sign
        // bit of its input (bit 7 of the input's top byte).
        uint32_t sgn[2];
        if constexpr (V == 8) {
            sgn[0] = __byte_perm(u.x, u.y, 0x7531);
            sgn[1] = __byte_perm(u.z, u.w, 0x7531);
        } else {
            sgn[0] = __byte_perm(__byte_perm(u.x, u.y, 0x0073), __byte_perm(u.z, u.w, 0x0073), 0x5410);
        }
#pragma unroll
        for (int w = 0; w < V / 4; ++w) {
            const uint32_t c0 = __nv_cvt_float2_to_fp8x2(q[2 * w], __NV_SATFINITE, __NV_E4M3);
            const uint32_t c1 = __nv_cvt_float2_to_fp8x2(q[2 * w + 1], __NV_SATFINITE, __NV_E4M3);
            words[w] = __byte_perm(c0, c1, 0x5410) | (sgn[w] & 0x80808080u);   // element 2h low in each half
        }
    } else {
        constexpr bool kClamp = OP == kOpActInt8Static || OP == kOpWeightAsym || DIRECT;
        const float2 M = splat2(kMagic), P = splat2(c.post);
        float2 t[V / 2];
#pragma unroll
        for (int e = 0; e < V / 2; ++e) {
            float2 x = q[e];
            if constexpr (kClamp) {
                x.x = clampf(x.x, c.qlo, c.qhi);
                x.y = clampf(x.y, c.qlo, c.qhi);
            }
            t[e] = __fadd2_rn(x, M);
            if constexpr (OP == kOpWeightAsym) t[e] = __fadd2_rn(t[e], P);
        }
        const uint32_t kp[2] = {keep.x, keep.y};
#pragma unroll
        for (int w = 0; w < V / 4; ++w)
            words[w] = pack_low_bytes(__float_as_uint(t[2 * w].x), __float_as_uint(t[2 * w].y),
                                      __float_as_uint(t[2 * w + 1].x), __float_as_uint(t[2 * w + 1].y)) &
                       kp[w];
    }
    return make_uint2(words[0], words[1]);
}

// Zeroes the 16-bit elements of a vector that are left out; mb holds 0xFF per
// left-out element.
__device__ __forceinline__ uint4 zero_skipped16(uint4 u, const uint2 mb) {
    // widen each mask byte to its 16-bit lane
    const uint32_t k0 = __byte_perm(mb.x, 0u, 0x1100), k1 = __byte_perm(mb.x, 0u, 0x3322);
    const uint32_t k2 = __byte_perm(mb.y, 0u, 0x1100), k3 = __byte_perm(mb.y, 0u, 0x3322);
    u.x &= ~k0; u.y &= ~k1; u.z &= ~k2; u.w &= ~k3;
    return u;
}

// Row min and max over one thread's vectors.  16-bit inputs (unsmoothed) keep
// packed 16-bit pairs, since min and max are exact in the input's own format,
// and widen to fp32 once per row.
template <typename T, int OP, bool PACKED = (sizeof(T) == 2 && OP != kOpActInt8Smooth)>
struct StatsAcc {
    float lo = FLT_MAX, hi = -FLT_MAX;
    __device__ __forceinline__ void add(const uint4 u, const float* mv = nullptr) {
        constexpr int V = VecOf<T>::N;
        float v[V];
        values_of<T, OP>(u, mv, v);
#pragma unroll
        for (int e = 0; e < V; ++e) {
            lo = fminf(lo, v[e]);
            hi = fmaxf(hi, v[e]);
        }
    }
    __device__ __forceinline__ RowStats get() const { return RowStats{0.f, lo, hi}; }
};

template <typename T, int OP>
struct StatsAcc<T, OP, true> {
    static constexpr bool kHalf = std::is_same<T, __half>::value;
    using T2 = typename std::conditional<kHalf, __half2, __nv_bfloat162>::type;
    // the largest finite value of T in both halves, and its negation
    uint32_t lo = kHalf ? 0x7BFF7BFFu : 0x7F7F7F7Fu;
    uint32_t hi = kHalf ? 0xFBFFFBFFu : 0xFF7FFF7Fu;
    __device__ __forceinline__ static T2 as2(uint32_t w) { return *reinterpret_cast<const T2*>(&w); }
    __device__ __forceinline__ static uint32_t bits(T2 v) { return *reinterpret_cast<const uint32_t*>(&v); }
    __device__ __forceinline__ void add(const uint4 u, const float* = nullptr) {
        const T2 a = as2(u.x), b = as2(u.y), c = as2(u.z), d = as2(u.w);
        hi = bits(__hmax2(as2(hi), __hmax2(__hmax2(a, b), __hmax2(c, d))));
        lo = bits(__hmin2(as2(lo), __hmin2(__hmin2(a, b), __hmin2(c, d))));
    }
    __device__ __forceinline__ RowStats get() const {
        const T2 h = as2(hi), l = as2(lo);
        return RowStats{0.f, fminf(static_cast<float>(l.x), static_cast<float>(l.y)),
                        fmaxf(static_cast<float>(h.x), static_cast<float>(h.y))};
    }
};

// The LLM.int8 outlier columns as one block sees them.  Thread i owns the
// run of `per` consecutive mask bytes from `begin`, held as bits; `before`
// outlier columns precede its run, `total` is the count.  A column's rank among
// the outliers (its slot in the gathered fp16 columns and in the ascending
// column list) is `before` plus the set bits below it in the run, so the
// gathers below scatter by rank and need no column list.
struct OutlierRuns {
    uint32_t bits[4];   // k <= 32768: runs of at most 128 columns
    int64_t begin;
    int per, before, total;
};

__device__ __forceinline__ OutlierRuns scan_outlier_mask(const uint8_t* mask, int64_t k, int* sh) {
    OutlierRuns r;
    // Runs of a multiple of 16 columns, read as 16-byte vectors (the mask is
    // 16-byte aligned and padded to the vector by the k % 32 == 0 rule).
    r.per = static_cast<int>((k + 16 * kBlock - 1) / (16 * kBlock)) * 16;
    r.begin = static_cast<int64_t>(threadIdx.x) * r.per;
    int local = 0;
#pragma unroll
    for (int w = 0; w < 4; ++w) r.bits[w] = 0u;
    for (int j0 = 0; j0 < r.per; j0 += 16) {
        const int64_t c0 = r.begin + j0;
        if (c0 >= k) break;
        const uint4 v = *reinterpret_cast<const uint4*>(mask + c0);
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int b = 0; b < 16; ++b) {
            if ((wv[b / 4] >> (8 * (b % 4))) & 0xFFu) {
                const int j = j0 + b;
                r.bits[j / 32] |= 1u << (j % 32);
                ++local;
            }
        }
    }
    // exclusive scan of `local` over the block
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) sh[warp] = incl;
    __syncthreads();
    int before_w = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kBlock / 32; ++w) {
        const int v = sh[w];
        if (w < warp) before_w += v;
        total += v;
    }
    __syncthreads();
    r.before = before_w + incl - local;
    r.total = total;
    return r;
}

// Outlier columns a block lists in shared memory (by rank) for its gathers;
// calls with more fall back to scattering from the mask runs.
constexpr int kSmemOutliers = 1024;

// Calls f(column, rank) for every outlier column of this thread's run.
template <typename F>
__device__ __forceinline__ void for_each_outlier(const OutlierRuns& r, F&& f) {
    int rank = r.before;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        uint32_t b = r.bits[w];
        while (b != 0u) {
            const int j = __ffs(b) - 1;
            b &= b - 1u;
            f(r.begin + 32 * w + j, rank++);
        }
    }
}

// One group of TPR (a multiple of 32) threads per row.  Thread t of a group
// handles the row's 16-byte vectors t, t + TPR, t + 2 TPR, ...; up to MAXV of
// them stay in registers between the two passes (longer rows are read twice,
// the second time from L2).
//
// PF (multi-wave matrices whose rows fit the register cache): the block
// walks its rows with a stride of the grid, and every thread issues the loads
// of its next row's vectors before it reduces and codes the current one, so
// HBM reads stay in flight through the reductions and the code pass.
template <typename T, int OP, int TPR, int MAXV, bool PF = false>
__global__ void __launch_bounds__(kBlock, PF ? (MAXV <= 4 ? 3 : 2) : (MAXV <= 4 ? 4 : 2))
row_quant_kernel(RowQuantArgs a) {
    static_assert(TPR % 32 == 0, "a warp works on one row");
    constexpr int V = VecOf<T>::N;
    constexpr int RPB = kBlock / TPR;
    constexpr bool kSkip = OP == kOpActInt8Skip;
    constexpr bool kRowsum = OP == kOpActInt8 || OP == kOpActInt8Skip || OP == kOpActInt8Static ||
                             OP == kOpActInt8Smooth;
    constexpr bool kSmooth = OP == kOpActInt8Smooth;
    __shared__ float red[3 * (kBlock / 32)];
    __shared__ int redi[kBlock / 32];
    __shared__ float cshare[kBlock / TPR][9];
    __shared__ int s_oidx[kSkip ? kSmemOutliers : 1];   // LLM.int8: outlier column of each rank

    const int g = threadIdx.x / TPR;
    const int t = threadIdx.x % TPR;
    const int64_t nvec = a.k / V;
    const bool cached = nvec <= static_cast<int64_t>(TPR) * MAXV;
    // Vectors this thread holds when the row is cached.
    const int nvl = cached ? static_cast<int>((nvec - t + TPR - 1) / TPR) : 0;
    const float bias = (OP == kOpWeightAsym && a.codes_u8) ? 128.0f : 0.0f;
    // Launched with programmatic dependent launch: this grid may start while
    // the previous kernel runs, so it waits for it before touching memory.
    // Activation quantizers first let the GEMM that follows launch, so that
    // its CTAs become resident and load their weights meanwhile (it waits for
    // this grid before reading the codes).  Weight quantizers do not: a GEMM
    // right after one must not load the weight before it is fully written.
    if constexpr (OP == kOpActInt8 || OP == kOpActInt8Skip || OP == kOpActFp8 || OP == kOpActInt8Static ||
                  OP == kOpActInt8Smooth)
        pdl_launch_dependents();
    pdl_wait();
    // PF: this thread's vectors of its group's next row (all rows are cached).
    uint4 nxt[PF ? MAXV : 1] = {};
    auto load_row = [&](int64_t r) {
        const T* p = static_cast<const T*>(a.src) + r * a.ld + static_cast<int64_t>(t) * V;
#pragma unroll
        for (int i = 0; i < MAXV; ++i)
            nxt[i] = i < nvl ? ld_stream16(p + i * TPR * V) : make_uint4(0u, 0u, 0u, 0u);
    };
    if constexpr (PF) {
        const int64_t r = static_cast<int64_t>(blockIdx.x) * RPB + g;
        if (r < a.rows) load_row(r);
    }

    // LLM.int8: rank the outlier columns; block 0 publishes the ascending
    // column list and the count (read by the GEMM that follows).
    OutlierRuns oruns;
    int cpad = 0;
    bool olist = false;   // the block's outlier columns are listed in s_oidx
    if constexpr (kSkip) {
        oruns = scan_outlier_mask(a.skip, a.k, redi);
        cpad = (oruns.total + 63) / 64 * 64;
        olist = oruns.total <= kSmemOutliers;
        if (olist) for_each_outlier(oruns, [&](int64_t c, int rank) { s_oidx[rank] = static_cast<int>(c); });
        if (blockIdx.x == 0) {
            for_each_outlier(oruns, [&](int64_t c, int rank) { a.outlier_idx[rank] = static_cast<int32_t>(c); });
            if (threadIdx.x == 0) *a.outlier_count = oruns.total;
        }
        __syncthreads();
    }

    for (int64_t row0 = static_cast<int64_t>(blockIdx.x) * RPB; row0 < a.rows;
         row0 += static_cast<int64_t>(gridDim.x) * RPB) {
        const int64_t row = row0 + g;
        const bool active = row < a.rows;   // the same for a whole warp
        const T* src_row = static_cast<const T*>(a.src) + (active ? row : 0) * a.ld;
        uint8_t* dst_row = static_cast<uint8_t*>(a.codes) + (active ? row : 0) * a.k;
        const T* src = src_row + static_cast<int64_t>(t) * V;
        uint8_t* dst = dst_row + static_cast<int64_t>(t) * V;
        const int nv = active ? nvl : 0;
        // Every thread of the block holds MAXV vectors: no per-vector guards.
        // (Uniform over the block, as the reductions below synchronize it.)
        const bool full = nvec == static_cast<int64_t>(TPR) * MAXV && row0 + RPB <= a.rows;
        auto keep_of = [&](int64_t j) -> uint2 {
            if constexpr (kSkip) {
                const uint2 m = *reinterpret_cast<const uint2*>(a.skip + j * V);
                return make_uint2(~(m.x * 0xFFu), ~(m.y * 0xFFu));
            } else {
                return make_uint2(~0u, ~0u);
            }
        };

        // Pass 1: row min and max (absmax = max(max, -min)).  Vectors past the
        // end of the row are zero, which leaves absmax unchanged; asymmetric
        // rows only count loaded vectors.  Left-out columns are zeroed.
        uint4 raw[MAXV];
        StatsAcc<T, OP> acc;
        if constexpr (PF) {
            // This row's vectors were loaded during the previous row; the next
            // row's loads go out now.
#pragma unroll
            for (int i = 0; i < MAXV; ++i) raw[i] = nxt[i];
            const int64_t rn = row + static_cast<int64_t>(gridDim.x) * RPB;
            if (rn < a.rows) load_row(rn);
        }
        auto pass1 = [&](auto full_tag) {
            constexpr bool FULL = decltype(full_tag)::value;
            if constexpr (!PF) {
#pragma unroll
                for (int i = 0; i < MAXV; ++i)
                    raw[i] = (FULL || i < nv) ? ld_stream16(src + i * TPR * V) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int i = 0; i < MAXV; ++i) {
                if (FULL || i < nv) {
                    if constexpr (kSkip) {
                        const uint2 kp = keep_of(t + static_cast<int64_t>(i) * TPR);
                        raw[i] = zero_skipped16(raw[i], make_uint2(~kp.x, ~kp.y));
                    }
                    if constexpr (kSmooth) {
                        float mv[V];
                        load_mult<V>(a.mult, t + static_cast<int64_t>(i) * TPR, mv);
                        acc.add(raw[i], mv);
                    } else {
                        acc.add(raw[i]);
                    }
                }
            }
        };
        if (cached) {
            if (full) pass1(std::true_type{}); else pass1(std::false_type{});
        } else if (active) {
            for (int64_t j = t; j < nvec; j += TPR) {
                uint4 u = ld_stream16(src_row + j * V);
                if constexpr (kSkip) {
                    const uint2 kp = keep_of(j);
                    u = zero_skipped16(u, make_uint2(~kp.x, ~kp.y));
                }
                if constexpr (kSmooth) {
                    float mv[V];
                    load_mult<V>(a.mult, j, mv);
                    acc.add(u, mv);
                } else {
                    acc.add(u);
                }
            }
        }
        RowStats st = acc.get();
        st.amax = fmaxf(st.hi, -st.lo);
        st = group_reduce<TPR, OP == kOpWeightAsym>(st, red);
        if constexpr (OP != kOpWeightAsym) st.amax = fmaxf(st.amax, 0.0f);

        RowConsts c;
        if constexpr (TPR > 32) {
            // One warp of the group works the row constants out for all.
            float* cs = cshare[g];
            if (t < 32) {
                c = row_consts<OP>(st.amax, st.lo, st.hi, a.clip_ub, bias, a.static_scale);
                if (t == 0) {
                    cs[0] = c.S; cs[1] = c.Z; cs[2] = c.bias; cs[3] = c.R;
                    cs[4] = c.qlo; cs[5] = c.qhi; cs[6] = c.post; cs[7] = c.direct ? 1.0f : 0.0f;
                    cs[8] = c.Rlo;
                }
            }
            group_sync<TPR>();
            c.S = cs[0]; c.Z = cs[1]; c.bias = cs[2]; c.R = cs[3];
            c.qlo = cs[4]; c.qhi = cs[5]; c.post = cs[6]; c.direct = cs[7] != 0.0f;
            c.Rlo = cs[8];
        } else {
            c = row_consts<OP>(st.amax, st.lo, st.hi, a.clip_ub, bias, a.static_scale);
        }

        // Pass 2: codes.  c.direct and `cached` are the same for the whole group.
        int rsum = 0;
        auto finish = [&](uint2 w, uint8_t* p) {
            if constexpr (V == 8) {
                *reinterpret_cast<uint2*>(p) = w;
            } else {
                *reinterpret_cast<uint32_t*>(p) = w.x;
            }
            if constexpr (kRowsum) {
                rsum = __dp4a(static_cast<int>(w.x), 0x01010101, rsum);
                if constexpr (V == 8) rsum = __dp4a(static_cast<int>(w.y), 0x01010101, rsum);
            }
        };
        auto pass2 = [&](auto full_tag) {
            constexpr bool FULL = decltype(full_tag)::value;
#pragma unroll
            for (int i = 0; i < MAXV; ++i) {
                if (FULL || i < nv) {
                    const int64_t j = t + static_cast<int64_t>(i) * TPR;
                    float mv[V];
                    if constexpr (kSmooth) load_mult<V>(a.mult, j, mv);
                    finish(code_vec<T, OP, false>(raw[i], c, keep_of(j), mv), dst + i * TPR * V);
                }
            }
        };
        if (cached && !c.direct) {
            if (full) pass2(std::true_type{}); else pass2(std::false_type{});
        } else if (active) {
            // Rows longer than the register cache (read again, from L2), and
            // rows coded with divisions.
            for (int64_t j = t; j < nvec; j += TPR) {
                const uint4 u = ld_stream16(src_row + j * V);
                float mv[V];
                if constexpr (kSmooth) load_mult<V>(a.mult, j, mv);
                const uint2 w = c.direct ? code_vec<T, OP, true>(u, c, keep_of(j), mv)
                                         : code_vec<T, OP, false>(u, c, keep_of(j), mv);
                finish(w, dst_row + j * V);
            }
        }
        if constexpr (kRowsum) rsum = group_sum<TPR>(rsum, redi);

        if (active && t == 0) {
            a.scale[row] = c.S;
            if constexpr (kRowsum) {
                if (a.rowsum) a.rowsum[row] = rsum;
            }
            if constexpr (OP == kOpWeightAsym) {
                a.zero_point[row] = a.codes_u8 ? __fadd_rn(c.Z, 128.0f) : c.Z;
            }
            if constexpr (OP == kOpWeightSym) {
                if (a.zero_point) a.zero_point[row] = 0.0f;
            }
        }
        // LLM.int8: gather the outlier columns of this iteration's rows into
        // fp16 by rank, zero-padded to a multiple of 64 columns for the
        // tensor-core outlier GEMM (the whole block works on each row).
        if constexpr (kSkip) {
            if (a.x_outlier != nullptr) {
                for (int i = 0; i < RPB; ++i) {
                    const int64_t r = row0 + i;
                    if (r >= a.rows) break;
                    const T* xs = static_cast<const T*>(a.src) + r * a.ld;
                    __half* xo = a.x_outlier + r * a.ldo;
                    if (olist) {
                        for (int j = static_cast<int>(threadIdx.x); j < cpad; j += kBlock)
                            xo[j] = j < oruns.total ? xs[s_oidx[j]] : __float2half_rn(0.0f);
                    } else {
                        for_each_outlier(oruns, [&](int64_t c, int rank) { xo[rank] = xs[c]; });
                        for (int j = oruns.total + static_cast<int>(threadIdx.x); j < cpad; j += kBlock)
                            xo[j] = __float2half_rn(0.0f);
                    }
                }
            }
        }
    }

    // LLM.int8: the fp16 outlier columns of the weight, by rank and
    // zero-padded like X's: W16's own columns, or the dequantized codes
    // fp16(fl32(S (q - Z))) when only the 8-bit weight is kept.
    if constexpr (kSkip) {
        auto w16_of = [&](int64_t r, int64_t c, float S, float Zr) -> __half {
            if (a.w16 != nullptr) return a.w16[r * a.w_ld + c];
            const float q = a.w_codes_u8
                                ? static_cast<float>(static_cast<const uint8_t*>(a.w_codes)[r * a.w_ld + c])
                                : static_cast<float>(static_cast<const int8_t*>(a.w_codes)[r * a.w_ld + c]);
            const float d = a.w_zero ? __fsub_rn(q, Zr) : q;
            return __float2half_rn(__fmul_rn(S, d));
        };
        if (olist) {
            // One weight row per warp at a time, so the rows' loads overlap.
            const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
            for (int64_t r = static_cast<int64_t>(blockIdx.x) * (kBlock / 32) + warp; r < a.w_rows;
                 r += static_cast<int64_t>(gridDim.x) * (kBlock / 32)) {
                __half* wo = a.w_outlier + r * a.ldo;
                const float S = a.w_scale[r];
                const float Zr = a.w_zero ? a.w_zero[r] : 0.0f;
                for (int j = lane; j < cpad; j += 32)
                    wo[j] = j < oruns.total ? w16_of(r, s_oidx[j], S, Zr) : __float2half_rn(0.0f);
            }
        } else {
            for (int64_t r = blockIdx.x; r < a.w_rows; r += gridDim.x) {
                __half* wo = a.w_outlier + r * a.ldo;
                const float S = a.w_scale[r];
                const float Zr = a.w_zero ? a.w_zero[r] : 0.0f;
                for_each_outlier(oruns, [&](int64_t c, int rank) { wo[rank] = w16_of(r, c, S, Zr); });
                for (int j = oruns.total + static_cast<int>(threadIdx.x); j < cpad; j += kBlock)
                    wo[j] = __float2half_rn(0.0f);
            }
        }
    }
}

template <typename T, int OP>
cudaError_t launch_rows_t(const RowQuantArgs& a, cudaStream_t s) {
    constexpr int V = VecOf<T>::N;
    const int64_t nvec = a.k / V;
    // PF launches a grid of at most 3 blocks per SM that strides over the rows.
    auto go = [&](auto tpr_tag, auto maxv_tag, auto pf_tag) -> cudaError_t {
        constexpr int TPR = decltype(tpr_tag)::value;
        constexpr int MAXV = decltype(maxv_tag)::value;
        constexpr bool PF = decltype(pf_tag)::value;
        constexpr int RPB = kBlock / TPR;
        int64_t blocks = (a.rows + RPB - 1) / RPB;
        if (blocks > 65535 * 4) blocks = 65535 * 4;
        if (PF) {
            int sms = 148, dev = 0;
            if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            const int per_sm = MAXV <= 4 ? 3 : 2;
            if (blocks > per_sm * sms) blocks = per_sm * sms;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
        cfg.blockDim = dim3(kBlock, 1, 1);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, row_quant_kernel<T, OP, TPR, MAXV, PF>, a);
    };
    using T128 = std::integral_constant<int, 128>;
    using T256 = std::integral_constant<int, 256>;
    using C2 = std::integral_constant<int, 2>;
    using C4 = std::integral_constant<int, 4>;
    using C16 = std::integral_constant<int, kMaxVec>;
    // Threads per row: enough to hold the row in registers (16 vectors a
    // thread), and, for short matrices, enough to spread the rows over the SMs;
    // otherwise as few as possible, so the per-row reductions (warp shuffles
    // for one warp) stay a small part of the work.
    const int64_t need = (nvec + kMaxVec - 1) / kMaxVec;
    const int64_t spread = (static_cast<int64_t>(kBlock) * 148 + a.rows - 1) / (a.rows > 0 ? a.rows : 1);
    int64_t tpr = need > spread ? need : spread;
    tpr = tpr <= 32 ? 32 : tpr <= 64 ? 64 : tpr <= 128 ? 128 : 256;
    // Matrices that take several waves of 16-vector rows run at 4 vectors a
    // thread instead (rows of up to 1024 vectors): fewer registers, twice the
    // resident warps, so loads of some rows overlap the arithmetic of others.
    const int64_t warps16 = a.rows * (tpr / 32);
    using Y = std::true_type;
    using N = std::false_type;
    // Multi-wave matrices: 8 vectors a thread (the per-row reductions and
    // constants are shared by twice the work of 4), the next row prefetched.
    if (warps16 > 2 * 148 * (kBlock / 32) && nvec <= 256 * 8) {
        using C8 = std::integral_constant<int, 8>;
        if (nvec <= 32 * 8) return go(std::integral_constant<int, 32>{}, C8{}, Y{});
        if (nvec <= 64 * 8) return go(std::integral_constant<int, 64>{}, C8{}, Y{});
        if (nvec <= 128 * 8) return go(T128{}, C8{}, Y{});
        return go(T256{}, C8{}, Y{});
    }
    // Rows spread over 128 or 256 threads hold a few vectors each: a kernel
    // unrolled for just those keeps the code short, which matters when each
    // SM runs it once (small batches: the instructions are fetched cold).
    if (tpr == 256 && nvec <= 256 * 2) return go(T256{}, C2{}, N{});
    // The LLM.int8 row pass also gathers the outlier columns of X and W by
    // block and by warp: one row per block gives those gathers twice the
    // blocks (512 x 4096 fp16: 32.1 -> 30.9 us per call).
    if (OP == kOpActInt8Skip && tpr >= 128 && nvec <= 256 * 2) return go(T256{}, C2{}, N{});
    if (tpr >= 128 && nvec <= 128 * 4) return go(T128{}, C4{}, N{});
    if (tpr == 256 && nvec <= 256 * 4) return go(T256{}, C4{}, N{});
    if (tpr == 32) return go(std::integral_constant<int, 32>{}, C16{}, N{});
    if (tpr == 64) return go(std::integral_constant<int, 64>{}, C16{}, N{});
    if (tpr == 128) return go(T128{}, C16{}, N{});
    return go(T256{}, C16{}, N{});
}

template <typename T>
cudaError_t launch_rows_dtype(const RowQuantArgs& a, cudaStream_t s) {
    switch (a.op) {
        case kOpActInt8:
            if (a.skip != nullptr) {
                if constexpr (std::is_same<T, __half>::value) return launch_rows_t<T, kOpActInt8Skip>(a, s);
                return cudaErrorInvalidValue;   // the outlier path takes fp16 inputs only
            }
            return launch_rows_t<T, kOpActInt8>(a, s);
        case kOpActFp8: return launch_rows_t<T, kOpActFp8>(a, s);
        case kOpActInt8Static: return launch_rows_t<T, kOpActInt8Static>(a, s);
        case kOpActInt8Smooth: return launch_rows_t<T, kOpActInt8Smooth>(a, s);
        case kOpWeightAsym: return launch_rows_t<T, kOpWeightAsym>(a, s);
        case kOpWeightSym: return launch_rows_t<T, kOpWeightSym>(a, s);
        case kOpWeightFp8: return launch_rows_t<T, kOpWeightFp8>(a, s);
    }
    return cudaErrorInvalidValue;
}

// ------------------------------------------------------------------ outliers

// Column absmax over all rows for a strip of 32 columns per block:
// 4 threads x 8 columns across the strip, 64 row lanes down it, eight rows'
// loads in flight per thread (512 rows per round).
template <typename T>
__global__ void __launch_bounds__(kBlock) outlier_colmax_kernel(const T* __restrict__ X, int64_t m,
                                                                int64_t k, int64_t ldx, float thr,
                                                                uint8_t* __restrict__ mask) {
    __shared__ float part[64][33];
    const int cv = threadIdx.x % 4;        // which 8-column vector of the strip
    const int rl = threadIdx.x / 4;        // row lane 0..63
    const int64_t col0 = static_cast<int64_t>(blockIdx.x) * 32 + cv * 8;
    // Launched with programmatic dependent launch: X may be the previous
    // kernel's output.  The row pass that follows may launch right away (it
    // waits for this grid before reading the mask).
    pdl_launch_dependents();
    pdl_wait();
    float mx[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) mx[e] = 0.f;
    if (col0 < k) {
        for (int64_t r0 = rl; r0 < m; r0 += 8 * 64) {
            uint4 u[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                u[i] = r0 + i * 64 < m ? ld_stream16(X + (r0 + i * 64) * ldx + col0) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float v[8];
                unpack_vec<T>(u[i], v);
#pragma unroll
                for (int e = 0; e < 8; ++e) mx[e] = fmaxf(mx[e], fabsf(v[e]));
            }
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) part[rl][cv * 8 + e] = mx[e];
    __syncthreads();
    // Two-level reduction of the 64 row lanes: each warp folds 8 of them for
    // the strip's 32 columns (independent loads), then one warp folds the 8.
    __shared__ float part2[8][32];
    {
        const int w = threadIdx.x / 32, c = threadIdx.x % 32;
        float v = 0.f;
#pragma unroll
        for (int r = 0; r < 8; ++r) v = fmaxf(v, part[w * 8 + r][c]);
        part2[w][c] = v;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        float c = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) c = fmaxf(c, part2[w][threadIdx.x]);
        const int64_t col = static_cast<int64_t>(blockIdx.x) * 32 + threadIdx.x;
        if (col < k) mask[col] = (thr > 0.f && c > thr) ? 1 : 0;
    }
}

__global__ void dequant_kernel(const void* __restrict__ codes, int code_dtype, int64_t n, int64_t k,
                               int64_t ldq, const float* __restrict__ S,
                               const float* __restrict__ Z, int out_dtype, void* __restrict__ out) {
    const int64_t total = n * k;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = i / k, c = i % k;
        float q;
        if (code_dtype == Q8_S8) q = static_cast<float>(static_cast<const int8_t*>(codes)[r * ldq + c]);
        else if (code_dtype == Q8_U8) q = static_cast<float>(static_cast<const uint8_t*>(codes)[r * ldq + c]);
        else {
            __nv_fp8_e4m3 f;
            f.__x = static_cast<const uint8_t*>(codes)[r * ldq + c];
            q = static_cast<float>(f);
        }
        const float d = Z ? __fsub_rn(q, Z[r]) : q;
        const float v = __fmul_rn(S[r], d);
        if (out_dtype == Q8_F32) static_cast<float*>(out)[i] = v;
        else if (out_dtype == Q8_F16) static_cast<__half*>(out)[i] = __float2half_rn(v);
        else static_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(v);
    }
}

}  // namespace

cudaError_t launch_row_quant(const RowQuantArgs& a, cudaStream_t s) {
    if (a.rows == 0) return cudaSuccess;
    switch (a.src_dtype) {
        case Q8_F16: return launch_rows_dtype<__half>(a, s);
        case Q8_BF16: return launch_rows_dtype<__nv_bfloat16>(a, s);
        case Q8_F32: return launch_rows_dtype<float>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_outlier_columns(const void* X, q8_dtype dt, int64_t m, int64_t k, int64_t ldx,
                                   float threshold, uint8_t* mask, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((k + 31) / 32), 1, 1);
    cfg.blockDim = dim3(kBlock, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (dt == Q8_F16)
        return cudaLaunchKernelEx(&cfg, outlier_colmax_kernel<__half>, static_cast<const __half*>(X), m, k, ldx,
                                  threshold, mask);
    return cudaLaunchKernelEx(&cfg, outlier_colmax_kernel<__nv_bfloat16>, static_cast<const __nv_bfloat16*>(X), m,
                              k, ldx, threshold, mask);
}

cudaError_t launch_dequant(const q8_weight& w, q8_dtype out_dtype, void* out, cudaStream_t s) {
    const int64_t total = w.n * w.k;
    if (total == 0) return cudaSuccess;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 148 * 32) blocks = 148 * 32;
    dequant_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
        w.codes, w.code_dtype, w.n, w.k, w.ld, w.scale, w.zero_point, out_dtype, out);
    return cudaGetLastError();
}

}  // namespace q8
