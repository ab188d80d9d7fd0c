// Grouped FP8 rowwise GEMM for mixture-of-experts layers on the sm_100a
// tensor cores.
//
// What is computed (Transformers FP8 / FBGEMM page, 5.4, Llama4 experts: the
// experts' FP8 weights sit in one tensor with per-row scales, and each
// expert's tokens are quantized and multiplied with f8f8bf16_rowwise on their
// own):
//   tokens are sorted by expert; rows offsets[e] .. offsets[e+1]-1 of the FP8
//   activation codes use expert e, whose weight is rows e*n .. e*n+n-1 of the
//   stacked E*n x k e4m3 weight;
//   acc = sum_k e4m3 x e4m3 (fp32 in TMEM), y = fl32(fl32(acc * Sx[m]) * Sw[e*n + j]),
//   y = fl32(y + bias[e*n + j]), Y = bf16(y).
//
// moe_fp8_kernel: one CTA per 128 x 128 output tile.  The grid holds an upper
// bound of the tiles, ceil(M / 128) + E rows of tiles (each expert adds at most
// one partial tile); each CTA finds its expert and first token from the
// device-side offsets (the routing result of the previous kernel) and leaves
// at once when its slot is past the last tile.  A tile's rows are read from
// the sorted activations at any row offset (TMA has no alignment rule for the
// outer coordinate) and rows past the expert's end are computed but not
// stored.  Warps: 0 TMA producer, 1 TMEM allocation + tcgen05.mma
// kind::f8f6f4, 2-5 epilogue.  No TMA multicast is used.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "q8_device.cuh"
#include "q8_internal.h"

namespace q8 {
namespace {

constexpr int kThreads = 192;
constexpr int kBM = 128;            // tokens per tile (MMA M, TMEM lanes)
constexpr int kBN = 128;            // output channels per tile (MMA N)
constexpr int kBKB = 128;           // bytes (= e4m3 values) of K per stage
constexpr int kABytes = kBM * kBKB;
constexpr int kBBytes = kBN * kBKB;
constexpr int kStage = kABytes + kBBytes;
constexpr int kStages = 6;
constexpr int kSmem = kStages * kStage + 1024;
constexpr int kTmemCols = kBN;

struct MoeParams {
    int m;                  // tokens (rows of the sorted activations)
    int n;                  // output channels per expert
    int experts;
    const int32_t* offsets; // [experts + 1]
    const float* sx;        // [m]
    const float* sw;        // [experts * n]
    const float* bias;      // [experts * n] or null
    __nv_bfloat16* y;
    int64_t ldy;
    int* status;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__global__ void __launch_bounds__(kThreads, 1)
moe_fp8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const MoeParams p, int num_kb) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full_bar[kStages];
    __shared__ __align__(8) uint64_t empty_bar[kStages];
    __shared__ __align__(8) uint64_t tfull_bar;
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    pdl_launch_dependents();
    pdl_wait();   // offsets, codes and scales come from the previous kernels

    // Slot blockIdx.y -> (expert, first token, end of the expert's tokens).
    // Offsets are clamped to [0, m] so that no tile reaches outside Y.
    int expert = -1, m0 = 0, m_end = 0;
    {
        int slot = static_cast<int>(blockIdx.y);
        int prev = p.offsets[0];
        prev = prev < 0 ? 0 : (prev > p.m ? p.m : prev);
        for (int e = 0; e < p.experts; ++e) {
            int hi = p.offsets[e + 1];
            hi = hi < prev ? prev : (hi > p.m ? p.m : hi);
            const int lo = prev;
            const int tiles = (hi - lo + kBM - 1) / kBM;
            if (slot < tiles) {
                expert = e;
                m0 = lo + slot * kBM;
                m_end = hi;
                break;
            }
            slot -= tiles;
            prev = hi;
        }
    }
    if (expert < 0) return;                        // past the last tile (uniform per CTA)
    const int n0 = static_cast<int>(blockIdx.x) * kBN;
    const int wrow0 = expert * p.n + n0;           // first stacked weight row of the tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&tfull_bar, 1);
        mbar_init(&drain_bar, 1);
        abort_sh = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;

    if (warp == 0) {
        if (elect_one()) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            uint32_t issued = 0, last_par = 0, phase = 0;
            int stage = 0;
            bool ok = true;
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_sh, p.status)) {
                    ok = false;
                    break;
                }
                uint8_t* sa = smem + stage * kStage;
                mbar_arrive_expect_tx(&full_bar[stage], kStage);
                tma_load_2d(sa, &tmA, &full_bar[stage], kb * kBKB, m0);
                tma_load_2d(sa + kABytes, &tmB, &full_bar[stage], kb * kBKB, wrow0);
                issued |= 1u << stage;
                last_par = (last_par & ~(1u << stage)) | (phase << stage);
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            if (!ok)
                for (int s = 0; s < kStages; ++s)
                    if (issued & (1u << s)) mbar_wait(&full_bar[s], (last_par >> s) & 1, nullptr, nullptr);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (elect_one()) {
            const uint32_t idesc = make_idesc(1, 0, 0, kBM, kBN);   // e4m3 x e4m3 -> f32
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!mbar_wait(&full_bar[stage], phase, &abort_sh, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = smem_addr(smem + stage * kStage);
                const uint64_t ad = sdesc_kmajor_sw128(sa);
                const uint64_t bd = sdesc_kmajor_sw128(sa + kABytes);
#pragma unroll
                for (int ks = 0; ks < kBKB / 32; ++ks)
                    mma_issue<kKindF8>(tmem_base, ad + 2 * ks, bd + 2 * ks, idesc, (kb | ks) != 0);
                tc_commit(&empty_bar[stage]);
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            tc_commit(ok ? &tfull_bar : &drain_bar);
            if (!ok) mbar_wait(&drain_bar, 0, nullptr, nullptr);
        }
        __syncwarp();
    } else {
        const int q = warp & 3;                    // TMEM lane quarter of this warp
        const int row = m0 + q * 32 + lane;
        const bool row_ok = row < m_end;
        const float sx = row_ok ? p.sx[row] : 0.f;
        const bool have = mbar_wait(&tfull_bar, 0, &abort_sh, p.status);
        if (have) tc_fence_after();
        const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
        for (int c = 0; c < kBN / 32; ++c) {
            __syncwarp();
            uint32_t r[32];
            tmem_ld32(tb + c * 32, r);
            tmem_ld_wait();
            const int n = n0 + c * 32;
            if (!have || !row_ok || n >= p.n) continue;
            const int nv = (p.n - n) >= 32 ? 32 : (p.n - n);   // 16 or 32 (n % 16 == 0)
            const float* sw = p.sw + static_cast<int64_t>(expert) * p.n + n;
            const float* bs = p.bias ? p.bias + static_cast<int64_t>(expert) * p.n + n : nullptr;
            float out[32];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (4 * j >= nv) break;
                const float4 s4 = *reinterpret_cast<const float4*>(sw + 4 * j);
                const float4 b4 = bs ? *reinterpret_cast<const float4*>(bs + 4 * j)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
                const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
                const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float v = __fmul_rn(__fmul_rn(__uint_as_float(r[4 * j + e]), sx), sv[e]);
                    if (bs) v = __fadd_rn(v, bv[e]);
                    out[4 * j + e] = v;
                }
            }
            uint4* yp = reinterpret_cast<uint4*>(p.y + static_cast<int64_t>(row) * p.ldy + n);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (8 * j >= nv) break;
                yp[j] = make_uint4(pack_bf16x2(out[8 * j], out[8 * j + 1]),
                                   pack_bf16x2(out[8 * j + 2], out[8 * j + 3]),
                                   pack_bf16x2(out[8 * j + 4], out[8 * j + 5]),
                                   pack_bf16x2(out[8 * j + 6], out[8 * j + 7]));
            }
        }
        __syncwarp();
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// K-major e4m3 rows with 128-byte swizzle, box of 128 bytes x `rows`.
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t k, uint64_t rows, uint64_t ld,
                 uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {k, rows};
    const cuuint64_t strides[1] = {ld};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBKB), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

q8_status launch_moe_fp8(const MoeArgs& a, cudaStream_t s) {
    if (a.m == 0 || a.n == 0 || a.experts == 0) return Q8_OK;
    // Persistent tile kernel with the expert-aware tile map when its map holds
    // the experts; else one CTA per 128 x 128 tile below.
    const q8_status st = launch_grouped_fp8(a, s);
    if (st != Q8_ERR_SHAPE) return st;
    CUtensorMap tA, tB;
    if (!make_map_u8(&tA, a.x_codes, a.k, a.m, a.ldx, kBM) ||
        !make_map_u8(&tB, a.w_codes, a.k, a.experts * a.n, a.ldw, kBN))
        return Q8_ERR_CUDA;
    if (cudaFuncSetAttribute(moe_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) !=
        cudaSuccess) {
        cudaGetLastError();
        return Q8_ERR_LAUNCH;
    }
    MoeParams p;
    p.m = static_cast<int>(a.m);
    p.n = static_cast<int>(a.n);
    p.experts = static_cast<int>(a.experts);
    p.offsets = a.offsets;
    p.sx = a.sx;
    p.sw = a.sw;
    p.bias = a.bias;
    p.y = a.y;
    p.ldy = a.ldy;
    p.status = device_status_ptr();
    const int tiles_n = static_cast<int>((a.n + kBN - 1) / kBN);
    const int slots = static_cast<int>((a.m + kBM - 1) / kBM + a.experts);
    const int num_kb = static_cast<int>((a.k + kBKB - 1) / kBKB);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles_n), static_cast<unsigned>(slots), 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, moe_fp8_kernel, tA, tB, p, num_kb) != cudaSuccess) {
        cudaGetLastError();
        return Q8_ERR_LAUNCH;
    }
    return Q8_OK;
}

}  // namespace q8
