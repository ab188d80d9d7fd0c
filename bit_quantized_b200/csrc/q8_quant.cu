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
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>
#include <type_traits>

#include "q8_device.cuh"
#include "q8_internal.h"

namespace q8 {
namespace {

constexpr float kEps = 1e-8f;
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
        __syncthreads();
        const int base = (warp / W) * W;
        RowStats r{0.f, FLT_MAX, -FLT_MAX};
#pragma unroll
        for (int i = 0; i < W; ++i) {
            r.amax = fmaxf(r.amax, red[3 * (base + i)]);
            r.lo = fminf(r.lo, red[3 * (base + i) + 1]);
            r.hi = fmaxf(r.hi, red[3 * (base + i) + 2]);
        }
        __syncthreads();
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
        __syncthreads();
        const int base = (warp / W) * W;
        int r = 0;
#pragma unroll
        for (int i = 0; i < W; ++i) r += red[base + i];
        __syncthreads();
        return r;
    }
    return v;
}

__device__ __forceinline__ float clampf(float v, float lo, float hi) {
    return fminf(fmaxf(v, lo), hi);
}


// Codes of one 16-byte vector (V elements) from the IEEE quotient fl32(x / S),
// without a division per element.
//
// With R = RN(1/S) (one reciprocal per row) the product t = RN(x * R) has a
// relative error below 2^-23 against x / S, and fl32(x / S) adds 2^-24, so
// |t - fl32(x / S)| <= 1.5 * 2^-23 |t|.
//   Integer codes: |t| <= 1024 (wider inputs are clamped; their codes saturate
//   anyway).  Adding 1.5 * 2^23 rounds t to an integer half to even (the sum lies
//   in [2^23, 2^24), where floats are integers, and the constant is even); the
//   low byte of the sum is the code's two's-complement byte (the constant's low
//   byte is 0), and d = t - rne(t) is exact.  An ulp of t is at most 2^-13, so
//   when |d| < 0.499 no half-integer lies between t and fl32(x / S): both round
//   to the same integer.
//   E4M3 codes: rounding to E4M3 (half to even, saturating) is monotonic, and
//   t (1 - 2^-20) and t (1 + 2^-20) bracket fl32(x / S); when both convert to
//   the same code, so does fl32(x / S).  (Values too small for the bracket to
//   widen round to zero either way.)
// A vector with any element near a rounding boundary is redone with exact
// divisions, out of line (it is rare).
constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23

__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
    return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

// Exact out-of-line paths; they take the packed input vector and return the
// packed codes by value so the fast paths keep everything in registers.
template <typename T>
__device__ __noinline__ uint2 int_codes_exact(const uint4 u, float S, float Z, float lo_clamp,
                                              float hi_clamp, float bias) {
    constexpr int V = VecOf<T>::N;
    float v[V];
    unpack_vec<T>(u, v);
    uint32_t words[2] = {0u, 0u};
    for (int w = 0; w < V / 4; ++w) {
        uint32_t b[4];
        for (int e = 0; e < 4; ++e) {
            float q = rintf(__fdiv_rn(v[4 * w + e], S));
            q = fminf(fmaxf(__fadd_rn(q, Z), lo_clamp), hi_clamp);
            b[e] = __float_as_uint(__fadd_rn(__fadd_rn(q, bias), kMagic));
        }
        words[w] = pack_low_bytes(b[0], b[1], b[2], b[3]);
    }
    return make_uint2(words[0], words[1]);
}

template <typename T>
__device__ __noinline__ uint2 e4m3_codes_exact(const uint4 u, float S) {
    constexpr int V = VecOf<T>::N;
    float v[V];
    unpack_vec<T>(u, v);
    uint32_t words[2] = {0u, 0u};
    for (int w = 0; w < V / 4; ++w) {
        uint32_t b[4];
        for (int e = 0; e < 4; ++e)
            b[e] = static_cast<uint32_t>(__nv_cvt_float_to_fp8(__fdiv_rn(v[4 * w + e], S), __NV_SATFINITE, __NV_E4M3));
        words[w] = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
    }
    return make_uint2(words[0], words[1]);
}

__device__ __forceinline__ float2 splat2(float a) { return make_float2(a, a); }

// The fast paths below work on pairs with the sm_100 packed fp32 instructions
// (two IEEE round-to-nearest operations per instruction, so each lane's result
// is the scalar one).

// Symmetric integer codes clamp(rne(x / S), -127, 127): |x / S| <= 127 up to
// rounding for every element of the row (the caller masks skipped columns).
template <typename T, int V>
__device__ __forceinline__ void int_codes_sym(const uint4 u, const float (&v)[V], float S, float R,
                                              uint32_t* words) {
    const float2 R2 = splat2(R), M2 = splat2(kMagic), nM2 = splat2(-kMagic), n1 = splat2(-1.0f);
    float dmax = 0.f;
#pragma unroll
    for (int w = 0; w < V / 4; ++w) {
        uint32_t b[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float2 t2 = __fmul2_rn(make_float2(v[4 * w + 2 * h], v[4 * w + 2 * h + 1]), R2);
            const float2 y2 = __fadd2_rn(t2, M2);
            const float2 d2 = __ffma2_rn(__fadd2_rn(y2, nM2), n1, t2);   // t - rne(t), exact
            dmax = fmaxf(dmax, fmaxf(fabsf(d2.x), fabsf(d2.y)));
            b[2 * h] = __float_as_uint(y2.x);
            b[2 * h + 1] = __float_as_uint(y2.y);
        }
        words[w] = pack_low_bytes(b[0], b[1], b[2], b[3]);
    }
    if (!(dmax < 0.499f)) {
        const uint2 r = int_codes_exact<T>(u, S, 0.0f, -127.0f, 127.0f, 0.0f);
        words[0] = r.x;
        if constexpr (V == 8) words[1] = r.y;
    }
}

// Asymmetric integer codes clamp(rne(x / S) + Z, -128, 127), + 128 for uint8.
template <typename T, int V>
__device__ __forceinline__ void int_codes_asym(const uint4 u, const float (&v)[V], float S, float R,
                                               float Z, float bias, uint32_t* words) {
    const float2 R2 = splat2(R), M2 = splat2(kMagic), nM2 = splat2(-kMagic), n1 = splat2(-1.0f);
    const float2 Z2 = splat2(Z), BM2 = splat2(bias + kMagic);
    float dmax = 0.f;
#pragma unroll
    for (int w = 0; w < V / 4; ++w) {
        uint32_t b[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float2 t2 = __fmul2_rn(make_float2(v[4 * w + 2 * h], v[4 * w + 2 * h + 1]), R2);
            t2.x = fminf(fmaxf(t2.x, -1024.0f), 1024.0f);
            t2.y = fminf(fmaxf(t2.y, -1024.0f), 1024.0f);
            const float2 q2 = __fadd2_rn(__fadd2_rn(t2, M2), nM2);
            const float2 d2 = __ffma2_rn(q2, n1, t2);
            dmax = fmaxf(dmax, fmaxf(fabsf(d2.x), fabsf(d2.y)));
            float2 c2 = __fadd2_rn(q2, Z2);
            c2.x = fminf(fmaxf(c2.x, -128.0f), 127.0f);
            c2.y = fminf(fmaxf(c2.y, -128.0f), 127.0f);
            const float2 e2 = __fadd2_rn(c2, BM2);   // integers below 2^23 + 2^8: exact
            b[2 * h] = __float_as_uint(e2.x);
            b[2 * h + 1] = __float_as_uint(e2.y);
        }
        words[w] = pack_low_bytes(b[0], b[1], b[2], b[3]);
    }
    if (!(dmax < 0.499f)) {
        const uint2 r = int_codes_exact<T>(u, S, Z, -128.0f, 127.0f, bias);
        words[0] = r.x;
        if constexpr (V == 8) words[1] = r.y;
    }
}

template <typename T, int V>
__device__ __forceinline__ void e4m3_codes(const uint4 u, const float (&v)[V], float S, float R,
                                           uint32_t* words) {
    const float2 R2 = splat2(R), lo2 = splat2(1.0f - 0x1p-20f), hi2 = splat2(1.0f + 0x1p-20f);
    bool bad = false;
#pragma unroll
    for (int w = 0; w < V / 4; ++w) {
        uint32_t hw[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float2 t2 = __fmul2_rn(make_float2(v[4 * w + 2 * h], v[4 * w + 2 * h + 1]), R2);
            const uint32_t cl = __nv_cvt_float2_to_fp8x2(__fmul2_rn(t2, lo2), __NV_SATFINITE, __NV_E4M3);
            const uint32_t ch = __nv_cvt_float2_to_fp8x2(__fmul2_rn(t2, hi2), __NV_SATFINITE, __NV_E4M3);
            bad |= cl != ch;
            hw[h] = cl;   // element 2h in the low byte, 2h + 1 in the high byte
        }
        words[w] = hw[0] | (hw[1] << 16);
    }
    if (bad) {
        const uint2 r = e4m3_codes_exact<T>(u, S);
        words[0] = r.x;
        if constexpr (V == 8) words[1] = r.y;
    }
}

// One group of TPR threads per row; up to MAXV 16-byte vectors per thread stay
// in registers between the two passes (longer rows are read twice, the second
// time from L2).
template <typename T, int OP, int TPR, int MAXV>
__global__ void __launch_bounds__(kBlock, 2) row_quant_kernel(RowQuantArgs a) {
    constexpr int V = VecOf<T>::N;
    constexpr int RPB = kBlock / TPR;
    __shared__ float red[3 * (kBlock / 32)];
    __shared__ int redi[kBlock / 32];

    const int g = threadIdx.x / TPR;
    const int t = threadIdx.x % TPR;
    const int64_t nvec = a.k / V;
    const bool cached = nvec <= static_cast<int64_t>(TPR) * MAXV;
    // Launched with programmatic dependent launch: this grid may start while
    // the previous kernel runs, so it waits for it before touching memory.
    // Activation quantizers then let the GEMM that follows start its prologue
    // and weight loads (it waits for this grid before reading the codes).
    // Weight quantizers do not: a GEMM right after one must not load the
    // weight before it is fully written.
    if constexpr (OP == kOpActInt8 || OP == kOpActFp8) pdl_launch_dependents();
    pdl_wait();

    for (int64_t row0 = static_cast<int64_t>(blockIdx.x) * RPB; row0 < a.rows;
         row0 += static_cast<int64_t>(gridDim.x) * RPB) {
        const int64_t row = row0 + g;
        const bool active = row < a.rows;
        const T* src = static_cast<const T*>(a.src) + (active ? row : 0) * a.ld;

        uint4 raw[MAXV];  // the row's 16-byte vectors, kept packed between the passes
        RowStats st{0.f, FLT_MAX, -FLT_MAX};
        const bool use_skip = (OP == kOpActInt8) && a.skip != nullptr;
        // Pass 1: row absmax (or min and max for the asymmetric scheme).  16-bit
        // inputs use packed pair min / max / abs, which are exact.
        auto accumulate = [&](const uint4 u, int64_t j) {
            if (use_skip) {
                float v[V];
                unpack_vec<T>(u, v);
#pragma unroll
                for (int e = 0; e < V; ++e)
                    if (a.skip[j * V + e] == 0) st.amax = fmaxf(st.amax, fabsf(v[e]));
            } else if constexpr (sizeof(T) == 2) {
                using T2 = typename std::conditional<std::is_same<T, __half>::value, __half2, __nv_bfloat162>::type;
                const T2* p2 = reinterpret_cast<const T2*>(&u);
                T2 m2 = p2[0];
                if constexpr (OP == kOpWeightAsym) {
                    T2 l2 = p2[0];
#pragma unroll
                    for (int q = 1; q < 4; ++q) {
                        m2 = __hmax2(m2, p2[q]);
                        l2 = __hmin2(l2, p2[q]);
                    }
                    st.hi = fmaxf(st.hi, fmaxf(static_cast<float>(m2.x), static_cast<float>(m2.y)));
                    st.lo = fminf(st.lo, fminf(static_cast<float>(l2.x), static_cast<float>(l2.y)));
                } else {
                    m2 = __habs2(m2);
#pragma unroll
                    for (int q = 1; q < 4; ++q) m2 = __hmax2(m2, __habs2(p2[q]));
                    st.amax = fmaxf(st.amax, fmaxf(static_cast<float>(m2.x), static_cast<float>(m2.y)));
                }
            } else {
                float v[V];
                unpack_vec<T>(u, v);
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    st.amax = fmaxf(st.amax, fabsf(v[e]));
                    st.lo = fminf(st.lo, v[e]);
                    st.hi = fmaxf(st.hi, v[e]);
                }
            }
        };
        if (active) {
            if (cached) {
                // All loads first, so they are in flight together.
#pragma unroll
                for (int i = 0; i < MAXV; ++i) {
                    const int64_t j = t + static_cast<int64_t>(i) * TPR;
                    if (j < nvec) raw[i] = ld_stream16(src + j * V);
                }
#pragma unroll
                for (int i = 0; i < MAXV; ++i) {
                    const int64_t j = t + static_cast<int64_t>(i) * TPR;
                    if (j < nvec) accumulate(raw[i], j);
                }
            } else {
                for (int64_t j = t; j < nvec; j += TPR) accumulate(ld_stream16(src + j * V), j);
            }
        }
        st = group_reduce<TPR, OP == kOpWeightAsym>(st, red);

        float S = 1.f, Z = 0.f;
        if constexpr (OP == kOpActInt8 || OP == kOpWeightSym) {
            S = __fdiv_rn(st.amax, 127.0f);
        } else if constexpr (OP == kOpActFp8 || OP == kOpWeightFp8) {
            float amax = st.amax;
            if (OP == kOpActFp8 && a.clip_ub > 0.f) amax = fminf(amax, a.clip_ub);
            S = __fdiv_rn(amax, 448.0f);
        } else {
            S = __fdiv_rn(__fsub_rn(st.hi, st.lo), 255.0f);
        }
        if (!(S >= kEps)) S = kEps;
        if constexpr (OP == kOpWeightAsym) {
            Z = clampf(__fsub_rn(rintf(__fdiv_rn(-st.lo, S)), 128.0f), -128.0f, 127.0f);
        }

        const float R = __frcp_rn(S);   // RN(1/S), shared by the row
        int rsum = 0;
        uint8_t* dst = static_cast<uint8_t*>(a.codes) + (active ? row : 0) * a.k;
        // Pass 2: codes (see int_codes_sym / int_codes_asym / e4m3_codes).
        auto quantize = [&](const uint4 u, int64_t j) {
            float v[V];
            unpack_vec<T>(u, v);
            uint32_t words[V / 4];
            if constexpr (OP == kOpActInt8 || OP == kOpWeightSym) {
                int_codes_sym<T, V>(u, v, S, R, words);
                if (use_skip) {
                    // LLM.int8: outlier columns carry code 0 (mask bytes are 0 or 1,
                    // so mask * 0xFF selects whole bytes).
#pragma unroll
                    for (int w = 0; w < V / 4; ++w)
                        words[w] &= ~(*reinterpret_cast<const uint32_t*>(a.skip + j * V + 4 * w) * 0xFFu);
                }
                if constexpr (OP == kOpActInt8) {
#pragma unroll
                    for (int w = 0; w < V / 4; ++w) rsum = __dp4a(static_cast<int>(words[w]), 0x01010101, rsum);
                }
            } else if constexpr (OP == kOpWeightAsym) {
                int_codes_asym<T, V>(u, v, S, R, Z, a.codes_u8 ? 128.0f : 0.0f, words);
            } else {
                e4m3_codes<T, V>(u, v, S, R, words);
            }
            if constexpr (V == 8) {
                *reinterpret_cast<uint2*>(dst + j * V) = make_uint2(words[0], words[1]);
            } else {
                *reinterpret_cast<uint32_t*>(dst + j * V) = words[0];
            }
        };
        if (active) {
            if (cached) {
#pragma unroll
                for (int i = 0; i < MAXV; ++i) {
                    const int64_t j = t + static_cast<int64_t>(i) * TPR;
                    if (j < nvec) quantize(raw[i], j);
                }
            } else {
                for (int64_t j = t; j < nvec; j += TPR) quantize(ld_stream16(src + j * V), j);
            }
        }
        if constexpr (OP == kOpActInt8) rsum = group_sum<TPR>(rsum, redi);

        if (active && t == 0) {
            a.scale[row] = S;
            if constexpr (OP == kOpActInt8) {
                if (a.rowsum) a.rowsum[row] = rsum;
            }
            if constexpr (OP == kOpWeightAsym) {
                a.zero_point[row] = a.codes_u8 ? __fadd_rn(Z, 128.0f) : Z;
            }
            if constexpr (OP == kOpWeightSym) {
                if (a.zero_point) a.zero_point[row] = 0.0f;
            }
        }
        // LLM.int8: gather the outlier columns of this row into fp16, zero-padded
        // to a multiple of 64 columns for the tensor-core outlier GEMM.
        if constexpr (OP == kOpActInt8 && sizeof(T) == 2) {
            if (active && a.x_outlier != nullptr) {
                const int cnt = *a.outlier_count;
                const int cpad = (cnt + 63) / 64 * 64;
                __half* xo = a.x_outlier + row * a.ldo;
                for (int j = t; j < cpad; j += TPR) {
                    __half h = __float2half_rn(0.0f);
                    if (j < cnt) {
                        const T x = src[a.outlier_idx[j]];
                        if constexpr (std::is_same<T, __half>::value) h = x;
                        else h = __float2half_rn(__bfloat162float(x));
                    }
                    xo[j] = h;
                }
            }
        }
    }
}

template <typename T, int OP>
cudaError_t launch_rows_t(const RowQuantArgs& a, cudaStream_t s) {
    constexpr int V = VecOf<T>::N;
    const int64_t nvec = a.k / V;
    // Threads per row: enough that each thread holds at most 8 vectors.
    auto go = [&](auto tpr_tag) -> cudaError_t {
        constexpr int TPR = decltype(tpr_tag)::value;
        constexpr int RPB = kBlock / TPR;
        int64_t blocks = (a.rows + RPB - 1) / RPB;
        if (blocks > 65535 * 4) blocks = 65535 * 4;
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
        return cudaLaunchKernelEx(&cfg, row_quant_kernel<T, OP, TPR, kMaxVec>, a);
    };
    // Threads per row: enough to hold the row in registers (16 vectors a
    // thread), and, for short matrices, enough to spread the rows over the SMs;
    // otherwise as few as possible, so the per-row reductions (warp shuffles
    // for one warp) stay a small part of the work.
    int64_t need = (nvec + kMaxVec - 1) / kMaxVec;
    int64_t spread = (static_cast<int64_t>(kBlock) * 148 + a.rows - 1) / (a.rows > 0 ? a.rows : 1);
    const int64_t tpr = need > spread ? need : spread;
    if (tpr <= 32) return go(std::integral_constant<int, 32>{});
    if (tpr <= 64) return go(std::integral_constant<int, 64>{});
    if (tpr <= 128) return go(std::integral_constant<int, 128>{});
    return go(std::integral_constant<int, 256>{});
}

template <typename T>
cudaError_t launch_rows_dtype(const RowQuantArgs& a, cudaStream_t s) {
    switch (a.op) {
        case kOpActInt8: return launch_rows_t<T, kOpActInt8>(a, s);
        case kOpActFp8: return launch_rows_t<T, kOpActFp8>(a, s);
        case kOpWeightAsym: return launch_rows_t<T, kOpWeightAsym>(a, s);
        case kOpWeightSym: return launch_rows_t<T, kOpWeightSym>(a, s);
        case kOpWeightFp8: return launch_rows_t<T, kOpWeightFp8>(a, s);
    }
    return cudaErrorInvalidValue;
}

// ------------------------------------------------------------------ outliers

// Column absmax over all rows for a strip of 32 columns per block:
// 4 threads x 8 columns across the strip, 64 row lanes down it.
template <typename T>
__global__ void __launch_bounds__(kBlock) outlier_colmax_kernel(const T* __restrict__ X, int64_t m,
                                                                int64_t k, int64_t ldx, float thr,
                                                                uint8_t* __restrict__ mask) {
    __shared__ float part[64][33];
    const int cv = threadIdx.x % 4;        // which 8-column vector of the strip
    const int rl = threadIdx.x / 4;        // row lane 0..63
    const int64_t col0 = static_cast<int64_t>(blockIdx.x) * 32 + cv * 8;
    float mx[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) mx[e] = 0.f;
    if (col0 < k) {
        for (int64_t r = rl; r < m; r += 64) {
            float v[8];
            load_vec<T>(X + r * ldx + col0, v);
#pragma unroll
            for (int e = 0; e < 8; ++e) mx[e] = fmaxf(mx[e], fabsf(v[e]));
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) part[rl][cv * 8 + e] = mx[e];
    __syncthreads();
    if (threadIdx.x < 32) {
        float c = 0.f;
        for (int r = 0; r < 64; ++r) c = fmaxf(c, part[r][threadIdx.x]);
        const int64_t col = static_cast<int64_t>(blockIdx.x) * 32 + threadIdx.x;
        if (col < k) mask[col] = (thr > 0.f && c > thr) ? 1 : 0;
    }
}

// Ordered compaction of the mask into idx[0..count): one block of 1024 threads,
// each owning a contiguous run of columns.
__global__ void __launch_bounds__(1024) outlier_scan_kernel(const uint8_t* __restrict__ mask,
                                                            int64_t k, int32_t* __restrict__ idx,
                                                            int32_t* __restrict__ count) {
    __shared__ int warp_tot[32];
    const int tid = threadIdx.x;
    const int64_t per = (k + 1023) / 1024;
    const int64_t b = tid * per, e = (b + per < k) ? b + per : k;
    int local = 0;
    for (int64_t c = b; c < e; ++c) local += mask[c] ? 1 : 0;
    // block exclusive scan of `local`
    const int lane = tid % 32, warp = tid / 32;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        warp_tot[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    int pos = incl - local + (warp > 0 ? warp_tot[warp - 1] : 0);
    for (int64_t c = b; c < e; ++c)
        if (mask[c]) idx[pos++] = static_cast<int32_t>(c);
    if (tid == 1023) *count = warp_tot[31];
}

// fp16 outlier columns of the weight: 256 threads per row, rows by blocks.
__global__ void __launch_bounds__(kBlock) gather_weight_outliers_kernel(
    const void* __restrict__ codes, int code_u8, int64_t ldq, const float* __restrict__ S,
    const float* __restrict__ Z, const __half* __restrict__ W16, int64_t n,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ count, __half* __restrict__ out,
    int64_t ldo) {
    const int cnt = *count;
    const int cpad = (cnt + 63) / 64 * 64;
    for (int64_t r = blockIdx.x; r < n; r += gridDim.x) {
        for (int j = threadIdx.x; j < cpad; j += blockDim.x) {
            __half h = __float2half_rn(0.0f);
            if (j < cnt) {
                const int64_t c = idx[j];
                if (W16 != nullptr) {
                    h = W16[r * ldq + c];
                } else {
                    const float q = code_u8 ? static_cast<float>(static_cast<const uint8_t*>(codes)[r * ldq + c])
                                            : static_cast<float>(static_cast<const int8_t*>(codes)[r * ldq + c]);
                    const float d = Z ? __fsub_rn(q, Z[r]) : q;
                    h = __float2half_rn(__fmul_rn(S[r], d));
                }
            }
            out[r * ldo + j] = h;
        }
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
                                   float threshold, uint8_t* mask, int32_t* idx, int32_t* count,
                                   cudaStream_t s) {
    const unsigned blocks = static_cast<unsigned>((k + 31) / 32);
    if (dt == Q8_F16)
        outlier_colmax_kernel<__half><<<blocks, kBlock, 0, s>>>(static_cast<const __half*>(X), m, k,
                                                                ldx, threshold, mask);
    else
        outlier_colmax_kernel<__nv_bfloat16><<<blocks, kBlock, 0, s>>>(
            static_cast<const __nv_bfloat16*>(X), m, k, ldx, threshold, mask);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    outlier_scan_kernel<<<1, 1024, 0, s>>>(mask, k, idx, count);
    return cudaGetLastError();
}

cudaError_t launch_gather_weight_outliers(const q8_weight& w, const __half* W16,
                                          const int32_t* idx, const int32_t* count, __half* W16o,
                                          int64_t ldo, cudaStream_t s) {
    int64_t blocks = w.n < 65535 ? w.n : 65535;
    gather_weight_outliers_kernel<<<static_cast<unsigned>(blocks), kBlock, 0, s>>>(
        w.codes, w.code_dtype == Q8_U8 ? 1 : 0, W16 ? w.k : w.ld, w.scale, w.zero_point, W16, w.n,
        idx, count, W16o, ldo);
    return cudaGetLastError();
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
