// W8A8 GEMMs on the sm_100a tensor cores (tcgen05) with TMEM accumulators,
// TMA-fed shared-memory pipelines and a fused dequant epilogue.
//
// What is computed ("大模型量化" (Xilyfe), INT32 accumulator section; the
// quantized matmul of the "大模型量化技术" overview, section 2.1, read with
// R = S (Q - Z); Transformers FP8 / FBGEMM page, section 5.3):
//   INT8  acc[m,n] = sum_k xq[m,k] wq[n,k]              (int32 in TMEM)
//         y = fl32(fl32(fl32(acc - Z[n] rowsum[m]) * Sx[m]) * Sw[n])
//   FP8   acc = sum_k e4m3 x e4m3                        (fp32 in TMEM)
//         y = fl32(fl32(acc * Sx[m]) * Sw[n])
//   LLM.int8 (bitsandbytes LLM.int8 page, 核心思想): a second fp32 TMEM
//         accumulator takes the fp16 outlier columns, y = fl32(y_int8 + y16)
//   then y = fl32(y + bias[n]) and Y = bf16_rne(y).
//
// Two kernels share the same warp roles (192 threads):
//   warp 0      TMA producer: one elected lane streams 128-byte-deep K slices
//               of both operands into a ring of shared-memory stages;
//   warp 1      allocates TMEM; one elected lane issues tcgen05.mma;
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (each warp reads its
//               own 32-lane quarter of TMEM), dequant, bf16 stores.
//
// gemm_tile_kernel    persistent over 128 x BN output tiles, activations as
//                     the MMA's M side; TMEM accumulators double-buffered so
//                     the epilogue of one tile overlaps the next tile's MMAs.
// gemm_decode_kernel  small token counts (decode): weights on the MMA's M side
//                     (128 output channels per CTA) and the tokens as N, with
//                     K split across the CTAs of a thread-block cluster whose
//                     partial accumulators are summed through distributed
//                     shared memory in a fixed rank order (exact for int32).
//
// No TMA multicast is used anywhere: each CTA loads its own tiles and the
// 126 MB L2 provides the reuse across CTAs.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <climits>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "q8_device.cuh"
#include "q8_internal.h"
#include "q8_qmath.cuh"

namespace q8 {
namespace {

constexpr int kBM = 128;        // MMA M (TMEM lanes)
constexpr int kBKB = 128;       // bytes of K per pipeline stage (one 128-byte swizzle row)
constexpr int kThreads = 192;
constexpr int kEpiStageBytes = 4 * 2 * 2048;   // output staging per CTA: 4 epilogue warps x 2 buffers
constexpr int kEpiConstBytes = 4 * 3 * 256 * 4; // column constants per CTA: 4 warps x 3 x BN (<= 256) floats
// Operand stages get what is left of the 227 KB a CTA may use once the
// epilogue's buffers, the 1 KB alignment slack and up to 5 KB of static
// shared memory (barriers, the grouped tile map) are set aside.
constexpr int kSmemBudget = 227 * 1024 - kEpiStageBytes - kEpiConstBytes - 1024 - 5 * 1024;

enum GemmKind { kS8S8 = 0, kS8U8 = 1, kE4M3 = 2 };

struct EpiParams {
    int m, n;
    const float* sx;
    const int32_t* rowsum;
    const float* sw;
    const float* zw;
    const float* bias;
    __nv_bfloat16* y;
    int64_t ldy;
    int8_t* yq;         // non-null: int8 output codes, clamp(rne(fl32(y / out_scale)), +-127)
    float out_scale;
    void* acc_debug;
    float* y16_debug;
    const int32_t* outlier_count;
    int* status;
};

template <int BN, bool MIXED>
struct TileCfg {
    static constexpr int A_BYTES = kBM * kBKB;
    static constexpr int B_BYTES = BN * kBKB;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int STAGES_RAW = kSmemBudget / STAGE;
    static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
    static constexpr int BUF_COLS = MIXED ? 2 * BN : BN;     // int32 acc (+ fp32 outlier acc)
    static constexpr int USED_COLS = 2 * BUF_COLS;
    static constexpr int TMEM_COLS = USED_COLS <= 32 ? 32 : USED_COLS <= 64 ? 64
                                   : USED_COLS <= 128 ? 128 : USED_COLS <= 256 ? 256 : 512;
    static constexpr int SMEM = STAGES * STAGE + kEpiStageBytes + kEpiConstBytes + 1024;
    static_assert(USED_COLS <= 512, "TMEM holds 512 columns");
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN");
};

template <int KIND>
constexpr uint32_t main_idesc(int n_mma) {
    // kind::i8: A = activations (s8), B = weights (s8 or u8), int32 accumulate.
    // kind::f8f6f4: both E4M3, fp32 accumulate.
    return KIND == kE4M3 ? make_idesc(1, 0, 0, kBM, n_mma)
                         : make_idesc(2, 1, KIND == kS8U8 ? 0 : 1, kBM, n_mma);
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Dequant of one accumulator value (int32 path): fl32(fl32(acc - Z rowsum) *
// Sx) * Sw, rounded once per step.  The zero-point correction is exact in
// 32-bit integers: Z (an integer in [-128, 255] held in fp32), Z rowsum,
// acc and their difference (= sum_k xq (wq - Z), at most 127 * 255 * K in
// magnitude) all stay below 2^31 for K <= 32768, and two's-complement
// subtraction gives the exact difference whenever that fits.
__device__ __forceinline__ float dequant_int(int32_t acc, float zw, int32_t rs, float sx, float sw,
                                             bool has_zp) {
    int32_t c = acc;
    if (has_zp) c -= __float2int_rn(zw) * rs;
    float v = __int2float_rn(c);
    v = __fmul_rn(v, sx);
    return __fmul_rn(v, sw);
}

// Re-quantized output code ("大模型量化" (Xilyfe), 量化对象 section: the INT32
// result is scaled back to INT8 before the next layer): the fp32 output y
// with the next layer's static scale S, clamp(rne(fl32(y / S)), -127, 127).
__device__ __forceinline__ uint32_t requant_code(float y, float S) {
    return static_cast<uint32_t>(static_cast<int>(fminf(fmaxf(rintf(__fdiv_rn(y, S)), -127.0f), 127.0f))) &
           0xFFu;
}

// The same code without a division per output.  y is clamped to
// [-128 S, 128 S] first (128 S is exact; codes beyond it saturate either way),
// so that q = RN(y / S) comes from R = RN(1/S) with qm::quotient (exact in
// that range), then q is clamped to [-127, 127] and rounded half to even by
// RN(q + 1.5 * 2^23), whose low byte is the code.  Scales below 2^-90 divide.
struct Requant {
    float S, R, T;
    bool direct;
};

__device__ __forceinline__ Requant requant_consts(float S) {
    Requant c;
    c.S = S;
    c.R = __frcp_rn(S);
    c.T = __fmul_rn(S, 128.0f);
    c.direct = !(S >= qm::kScaleMin);
    return c;
}

// Out of line: the unrolled epilogue stays short (it shares the instruction
// cache with the MMA warp's loop).
__device__ __noinline__ uint32_t requant_code_slow(float y, float S) { return requant_code(y, S); }

__device__ __forceinline__ uint32_t requant_code_fast(float y, const Requant& c) {
    if (c.direct) return requant_code_slow(y, c.S);
    const float q = qm::quotient(fminf(fmaxf(y, -c.T), c.T), c.S, c.R);
    return __float_as_uint(__fadd_rn(fminf(fmaxf(q, -127.0f), 127.0f), qm::kMagic)) & 0xFFu;
}

// Codes of 4 outputs, packed in order.
__device__ __forceinline__ uint32_t requant_codes4(const float* y, const Requant& c) {
    uint32_t w = 0u;
#pragma unroll
    for (int e = 0; e < 4; ++e) w |= requant_code_fast(y[e], c) << (8 * e);
    return w;
}

// bf16_rne(a) in the low half, bf16_rne(b) in the high half (one conversion).
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// Output path of the bf16 epilogue.  With a tensor map, each warp stages its
// 32 x 32 output chunk (rows of 64 bytes, 16-byte chunks swizzled by
// (row / 2) % 4, which is TMA's 64-byte swizzle and keeps the 32 lanes' writes
// free of bank conflicts) in one of two 2 KB buffers of its own, and one lane
// stores it with a TMA tensor store that clips rows and columns past the
// output.  The store runs asynchronously, so it overlaps the next chunk and the
// next tile, and writes whole sectors, where 32 lanes storing 16 bytes of 32
// different rows would each leave a partial one.  Without a tensor map (the
// INT8-output epilogue, or no map) every thread stores its own row directly.
struct EpiStore {
    const CUtensorMap* tmY;   // null: direct stores
    uint8_t* stage;           // this warp's 2 x 2048 bytes (1024-aligned)
    int row0;                 // first output row of this warp's 32
    uint32_t* sbuf;           // which of the two buffers is next
    const float* colc;        // this tile's weight scales, zero points, bias: 3 x BN (shared)
    float sx;                 // this thread's row: token scale
    int32_t rs;               //                    and row sum
    int row_end;              // rows >= row_end are not stored
    bool tma_tile;            // this warp's 32 rows may go through the tensor store
};

// The column and row constants of a tile, fetched into registers a tile
// ahead: every lane holds BN / 32 columns of each constant.  The epilogue of
// the current tile then reads them from warp-private shared memory (one
// broadcast load per four columns) instead of waiting on global loads.
template <int BN>
struct EpiConsts {
    float c[3][BN / 32];
    float sx;
    int32_t rs;

    // Columns n_tile.. of the output (col_off + column in the scale and bias
    // arrays), and this thread's row (stored only below row_end).
    __device__ __forceinline__ void fetch(const EpiParams& p, int n_tile, int col_off, int row,
                                          int row_end) {
        const int lane = threadIdx.x % 32;
#pragma unroll
        for (int i = 0; i < BN / 32; ++i) {
            const int col = n_tile + i * 32 + lane;
            const bool ok = col < p.n;
            c[0][i] = ok ? p.sw[col_off + col] : 0.f;
            c[1][i] = (ok && p.zw) ? p.zw[col_off + col] : 0.f;
            c[2][i] = (ok && p.bias) ? p.bias[col_off + col] : 0.f;
        }
        const bool rok = row < row_end;
        sx = rok ? p.sx[row] : 0.f;
        rs = (rok && p.zw && p.rowsum) ? p.rowsum[row] : 0;
    }

    // Publishes the column constants to the warp's shared array (3 x BN).
    __device__ __forceinline__ void publish(float* colc) const {
        const int lane = threadIdx.x % 32;
        __syncwarp();
#pragma unroll
        for (int i = 0; i < BN / 32; ++i) {
            colc[i * 32 + lane] = c[0][i];
            colc[BN + i * 32 + lane] = c[1][i];
            colc[2 * BN + i * 32 + lane] = c[2][i];
        }
        __syncwarp();
    }
};


__device__ __forceinline__ void st_shared_v4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(smem_addr(p)), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

// Dequant epilogue of one accumulator tile for the calling thread's output
// row: BN columns from n_tile, read from TMEM at `tb` (the warp's 32-lane
// quarter and the accumulator buffer); the LLM.int8 outlier accumulator sits
// BN columns further.  Every thread of the warp calls it (tcgen05.ld is
// warp-wide); rows and columns past the output are computed and not stored.
template <int BN, int KIND, bool MIXED, bool QOUT>
__device__ __forceinline__ void epilogue_tile(const EpiParams& p, uint32_t tb, int row, int n_tile,
                                              int n16_kb, const EpiStore& es) {
    const int lane = threadIdx.x % 32;
    const bool has_zp = p.zw != nullptr;
    const bool row_ok = row < es.row_end;
    const float sx = es.sx;
    const int32_t rs = es.rs;
    const bool tma = !QOUT && es.tmY != nullptr && es.tma_tile;
    // Accumulator columns are read from TMEM G chunks of 32 at a time.
    constexpr int NCH = BN / 32;
    constexpr int G = 1;
#pragma unroll 1
    for (int c0 = 0; c0 < NCH; c0 += G) {
        __syncwarp();
        uint32_t rg[G][32];
#pragma unroll
        for (int g = 0; g < G; ++g)
            if (c0 + g < NCH) tmem_ld32(tb + (c0 + g) * 32, rg[g]);
        uint32_t r16[32];
        if constexpr (MIXED) {
            if (n16_kb > 0) tmem_ld32(tb + BN + c0 * 32, r16);
        }
        tmem_ld_wait();
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const int c = c0 + g;
        if (c >= NCH) break;
        const uint32_t (&r)[32] = rg[g];
        const int n0 = n_tile + c * 32;
        if (n0 >= p.n) continue;                               // uniform over the warp
        const int nv = (p.n - n0) >= 32 ? 32 : (p.n - n0);   // 16 or 32
        float out[32];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (4 * j >= nv) break;
            const float* cc = es.colc + c * 32 + 4 * j;
            const float4 sw4 = *reinterpret_cast<const float4*>(cc);
            float4 zw4 = make_float4(0.f, 0.f, 0.f, 0.f), b4 = zw4;
            if (has_zp) zw4 = *reinterpret_cast<const float4*>(cc + BN);
            if (p.bias) b4 = *reinterpret_cast<const float4*>(cc + 2 * BN);
            const float swv[4] = {sw4.x, sw4.y, sw4.z, sw4.w};
            const float zwv[4] = {zw4.x, zw4.y, zw4.z, zw4.w};
            const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = 4 * j + e;
                float v;
                if constexpr (KIND == kE4M3) {
                    v = __fmul_rn(__fmul_rn(__uint_as_float(r[i]), sx), swv[e]);
                } else {
                    v = dequant_int(static_cast<int32_t>(r[i]), zwv[e], rs, sx, swv[e], has_zp);
                }
                if constexpr (MIXED) {
                    const float y16 = n16_kb > 0 ? __uint_as_float(r16[i]) : 0.0f;
                    v = __fadd_rn(v, y16);
                }
                if (p.bias) v = __fadd_rn(v, bv[e]);
                out[i] = v;
            }
        }
        if (tma) {
            uint8_t* buf = es.stage + *es.sbuf * 2048;
            if (lane == 0) bulk_wait_read<1>();   // the buffer's previous store has read it
            __syncwarp();
            const uint32_t sw = static_cast<uint32_t>((lane >> 1) & 3);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (8 * j < nv)
                    st_shared_v4(buf + lane * 64 + ((static_cast<uint32_t>(j) ^ sw) << 4),
                                 pack_bf16(out[8 * j], out[8 * j + 1]),
                                 pack_bf16(out[8 * j + 2], out[8 * j + 3]),
                                 pack_bf16(out[8 * j + 4], out[8 * j + 5]),
                                 pack_bf16(out[8 * j + 6], out[8 * j + 7]));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_2d(es.tmY, buf, n0, es.row0);
                bulk_commit();
            }
            *es.sbuf ^= 1u;
        } else if (row_ok) {
            if constexpr (QOUT) {
                const Requant rq = requant_consts(p.out_scale);
                uint32_t w[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) w[j] = requant_codes4(&out[4 * j], rq);
                uint4* qp = reinterpret_cast<uint4*>(p.yq + static_cast<int64_t>(row) * p.ldy + n0);
                qp[0] = make_uint4(w[0], w[1], w[2], w[3]);
                if (nv > 16) qp[1] = make_uint4(w[4], w[5], w[6], w[7]);
            } else {
                uint4* yp = reinterpret_cast<uint4*>(p.y + static_cast<int64_t>(row) * p.ldy + n0);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (8 * j >= nv) break;
                    yp[j] = make_uint4(pack_bf16(out[8 * j], out[8 * j + 1]),
                                       pack_bf16(out[8 * j + 2], out[8 * j + 3]),
                                       pack_bf16(out[8 * j + 4], out[8 * j + 5]),
                                       pack_bf16(out[8 * j + 6], out[8 * j + 7]));
                }
            }
        }
        if (row_ok && p.acc_debug) {
            uint4* ap = reinterpret_cast<uint4*>(static_cast<uint32_t*>(p.acc_debug) +
                                                 static_cast<int64_t>(row) * p.n + n0);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (4 * j >= nv) break;
                ap[j] = make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
            }
        }
        if constexpr (MIXED) {
            if (row_ok && p.y16_debug) {
                uint4* dp = reinterpret_cast<uint4*>(p.y16_debug + static_cast<int64_t>(row) * p.n + n0);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (4 * j >= nv) break;
                    if (n16_kb > 0)
                        dp[j] = make_uint4(r16[4 * j], r16[4 * j + 1], r16[4 * j + 2], r16[4 * j + 3]);
                    else
                        dp[j] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
        }
    }
    }
}

// Where one output tile of a persistent schedule lies.
struct TileRef {
    int a_row;     // first activation row the tile reads
    int row_end;   // rows at or past row_end are computed and not stored
    int b_row;     // first weight row
    int n_tile;    // first output column
    int col_off;   // offset of the output columns in the scale and bias arrays
};

// Dense schedule: tiles_m x tiles_n tiles, the M index fastest.
__device__ __forceinline__ TileRef dense_tile(int tile, int tiles_m, int rows, int bn, int m) {
    const int tm = tile % tiles_m, tn = tile / tiles_m;
    return TileRef{tm * rows, m, tn * bn, tn * bn, 0};
}

// Grouped schedule of a mixture-of-experts layer (the grouped FP8 linear of
// the FBGEMM FP8 page, section 5.4): tokens sorted by expert, rows
// off[e] .. off[e+1]-1 meet expert e's weight rows e*n .. e*n+n-1.  Expert e
// has ceil((off[e+1] - off[e]) / rows) row tiles; mt[e] counts those of the
// experts before it, so the layer has mt[E] x tiles_n tiles, the row-tile index
// fastest.  A tile starts at any token row (TMA has no alignment rule for the
// outer coordinate); rows past the expert's end are computed and not stored.
constexpr int kMaxGroupedExperts = 512;

__device__ __forceinline__ TileRef grouped_tile(int tile, const int* off, const int* mt, int experts,
                                                int rows, int bn, int n) {
    const int G = mt[experts];
    const int g = tile % G, tn = tile / G;
    // the expert e with mt[e] <= g < mt[e + 1] (empty experts have none)
    int lo = 0, hi = experts;   // mt[lo] <= g < mt[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (mt[mid] <= g) lo = mid; else hi = mid;
    }
    return TileRef{off[lo] + (g - mt[lo]) * rows, off[lo + 1], lo * n + tn * bn, tn * bn, lo * n};
}

// off[0..E]: the offsets clamped to [0, m] and made non-decreasing; mt[0..E]:
// the row-tile prefix.  One warp, 32 experts at a time.
__device__ __forceinline__ void build_group_map(const int32_t* offsets, int experts, int m, int rows,
                                                int* off, int* mt) {
    const int lane = threadIdx.x % 32;
    int carry_off = 0, carry_mt = 0;
    for (int base = 0; base <= experts; base += 32) {
        const int e = base + lane;
        int v = e <= experts ? offsets[e] : m;
        v = v < 0 ? 0 : (v > m ? m : v);
        v = v > carry_off ? v : carry_off;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {   // running maximum
            const int y = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v = v > y ? v : y;
        }
        // expert e - 1 spans [off[e - 1], off[e]): its row tiles, counted at index e
        const int prev = __shfl_up_sync(0xffffffffu, v, 1);
        const int lo_e = lane == 0 ? carry_off : prev;
        int t = (e >= 1 && e <= experts) ? (v - lo_e + rows - 1) / rows : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {   // inclusive sum
            const int y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        if (e <= experts) {
            off[e] = v;
            mt[e] = carry_mt + t;
        }
        carry_off = __shfl_sync(0xffffffffu, v, 31);
        carry_mt += __shfl_sync(0xffffffffu, t, 31);
    }
}

// ============================================================================
// Persistent tile kernel
// ============================================================================
template <int BN, int KIND, bool MIXED, bool QOUT, bool GROUPED = false>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tile_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmA16,
                 const __grid_constant__ CUtensorMap tmB16, const __grid_constant__ CUtensorMap tmY,
                 int use_tmy, const EpiParams p, int num_kb, int tiles_m, int tiles_n,
                 const int32_t* group_offsets, int experts) {
    using C = TileCfg<BN, MIXED>;
    static_assert(!(GROUPED && MIXED), "grouped tiles carry no outlier stream");
    __shared__ int g_off[GROUPED ? kMaxGroupedExperts + 1 : 1];
    __shared__ int g_mt[GROUPED ? kMaxGroupedExperts + 1 : 1];
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    __shared__ __align__(8) uint64_t full_bar[C::STAGES];
    __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull_bar[b], 1);
            mbar_init(&tempty_bar[b], 4);
        }
        mbar_init(&drain_bar, 1);
        abort_sh = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, C::TMEM_COLS);
        tmem_relinquish();
    }
    if constexpr (GROUPED) {
        // The routing offsets come from the previous kernels.
        pdl_wait();
        if (warp == 2) build_group_map(group_offsets, experts, p.m, kBM, g_off, g_mt);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;
    // The next kernel (typically the next layer's activation quantizer, which
    // waits for this grid before touching memory) may launch now.
    pdl_launch_dependents();

    int n16_kb = 0;
    if constexpr (MIXED) {
        // The outlier count comes from the previous kernels (the producer
        // reads it after its early weight loads).
        if (warp != 0) {
            pdl_wait();
            n16_kb = (*p.outlier_count + 63) / 64;
        }
    }
    const int total_kb = num_kb + n16_kb;
    const int num_tiles = GROUPED ? g_mt[GROUPED ? experts : 0] * tiles_n : tiles_m * tiles_n;
    auto tile_ref = [&](int tile) -> TileRef {
        if constexpr (GROUPED) return grouped_tile(tile, g_off, g_mt, experts, kBM, BN, p.n);
        else return dense_tile(tile, tiles_m, kBM, BN, p.m);
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (elect_one()) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            if constexpr (MIXED) {
                tma_prefetch_desc(&tmA16);
                tma_prefetch_desc(&tmB16);
            }
            // The weights do not depend on the previous kernel (a weight
            // quantizer lets no dependent grid start before it completes): the
            // first ring of the first tile's weight slices goes out before the
            // programmatic-launch wait, the activation slices after it.
            int npre = 0;
            if constexpr (!GROUPED) {
                if (static_cast<int>(blockIdx.x) < num_tiles) {
                    const TileRef tr0 = tile_ref(blockIdx.x);
                    npre = num_kb < C::STAGES ? num_kb : C::STAGES;
                    for (int s = 0; s < npre; ++s) {
                        mbar_arrive_expect_tx(&full_bar[s], C::STAGE);
                        tma_load_2d(smem + s * C::STAGE + C::A_BYTES, &tmB, &full_bar[s], s * kBKB, tr0.b_row);
                    }
                }
            }
            pdl_wait();   // operands may come from the previous kernel
            int ptotal_kb = total_kb;
            if constexpr (MIXED) ptotal_kb = num_kb + (*p.outlier_count + 63) / 64;
            uint32_t issued = 0;             // stages that ever received a load
            uint32_t last_par = 0;           // parity of each stage's last load
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const TileRef tr = tile_ref(tile);
                for (int kb = 0; kb < ptotal_kb; ++kb) {
                    const bool pre = tile == static_cast<int>(blockIdx.x) && kb < npre;   // weight already out
                    if (!pre && !mbar_wait(&empty_bar[stage], phase ^ 1, &abort_sh, p.status)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + stage * C::STAGE;
                    uint8_t* sb = sa + C::A_BYTES;
                    if (!pre) mbar_arrive_expect_tx(&full_bar[stage], C::STAGE);
                    if (!MIXED || kb < num_kb) {
                        tma_load_2d(sa, &tmA, &full_bar[stage], kb * kBKB, tr.a_row);
                        if (!pre) tma_load_2d(sb, &tmB, &full_bar[stage], kb * kBKB, tr.b_row);
                    } else {
                        const int k16 = (kb - num_kb) * 64;
                        tma_load_2d(sa, &tmA16, &full_bar[stage], k16, tr.a_row);
                        tma_load_2d(sb, &tmB16, &full_bar[stage], k16, tr.b_row);
                    }
                    issued |= 1u << stage;
                    last_par = (last_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            if (!ok) {
                // Abort: let every load already issued land before the CTA exits.
                for (int s = 0; s < C::STAGES; ++s)
                    if (issued & (1u << s)) mbar_wait(&full_bar[s], (last_par >> s) & 1, nullptr, nullptr);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (elect_one()) {
            const uint32_t idesc = main_idesc<KIND>(BN);
            const uint32_t idesc16 = make_idesc(1, 0, 0, kBM, BN);  // f16 x f16 -> f32
            int stage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t bphase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                if (!mbar_wait(&tempty_bar[buf], bphase ^ 1, &abort_sh, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_main = tmem_base + buf * C::BUF_COLS;
                for (int kb = 0; kb < total_kb; ++kb) {
                    if (!mbar_wait(&full_bar[stage], phase, &abort_sh, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_addr(smem + stage * C::STAGE);
                    const uint64_t ad = sdesc_kmajor_sw128(sa);
                    const uint64_t bd = sdesc_kmajor_sw128(sa + C::A_BYTES);
                    if (!MIXED || kb < num_kb) {
#pragma unroll
                        for (int ks = 0; ks < kBKB / 32; ++ks) {
                            if constexpr (KIND == kE4M3)
                                mma_issue<kKindF8>(d_main, ad + 2 * ks, bd + 2 * ks, idesc, (kb | ks) != 0);
                            else
                                mma_issue<kKindI8>(d_main, ad + 2 * ks, bd + 2 * ks, idesc, (kb | ks) != 0);
                        }
                    } else {
#pragma unroll
                        for (int ks = 0; ks < kBKB / 32; ++ks)
                            mma_issue<kKindF16>(d_main + BN, ad + 2 * ks, bd + 2 * ks, idesc16,
                                                ((kb - num_kb) | ks) != 0);
                    }
                    tc_commit(&empty_bar[stage]);
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                tc_commit(&tfull_bar[buf]);
                buf ^= 1;
                if (buf == 0) bphase ^= 1;
            }
            if (!ok) {
                // Abort: wait for the MMAs already issued before TMEM is freed.
                tc_commit(&drain_bar);
                mbar_wait(&drain_bar, 0, nullptr, nullptr);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue
        pdl_wait();   // scales and row sums may come from the previous kernel
        const int q = warp & 3;  // this warp's TMEM lane quarter
        uint32_t sbuf = 0;
        uint8_t* epi_smem = smem + C::STAGES * C::STAGE;
        float* colc = reinterpret_cast<float*>(epi_smem + kEpiStageBytes) + (warp - 2) * 3 * BN;
        EpiStore es{use_tmy ? &tmY : nullptr, epi_smem + (warp - 2) * 4096, 0, &sbuf, colc, 0.f, 0, 0,
                    false};
        EpiConsts<BN> pf;
        if (static_cast<int>(blockIdx.x) < num_tiles) {
            const TileRef t0 = tile_ref(static_cast<int>(blockIdx.x));
            pf.fetch(p, t0.n_tile, t0.col_off, t0.a_row + q * 32 + lane, t0.row_end);
        }
        int buf = 0;
        uint32_t bphase = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const TileRef tr = tile_ref(tile);
            if (!mbar_wait(&tfull_bar[buf], bphase, &abort_sh, p.status)) break;
            tc_fence_after();
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * C::BUF_COLS;
            es.row0 = tr.a_row + q * 32;
            es.row_end = tr.row_end;
            // A tensor store clips at the output's last row only: chunks that
            // cross an expert's end are stored row by row.
            es.tma_tile = GROUPED ? es.row0 + 32 <= tr.row_end : es.row0 < tr.row_end;
            pf.publish(colc);
            es.sx = pf.sx;
            es.rs = pf.rs;
            const int nt = tile + static_cast<int>(gridDim.x);
            if (nt < num_tiles) {
                const TileRef tn = tile_ref(nt);
                pf.fetch(p, tn.n_tile, tn.col_off, tn.a_row + q * 32 + lane, tn.row_end);
            }
            epilogue_tile<BN, KIND, MIXED, QOUT>(p, tb, es.row0 + lane, tr.n_tile, n16_kb, es);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty_bar[buf]);
            buf ^= 1;
            if (buf == 0) bphase ^= 1;
        }
        if (lane == 0) bulk_wait_all();   // staged output stores done before the CTA ends
        __syncwarp();
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ============================================================================
// Persistent pair kernel: 256 x BN tiles on the two SMs of a CTA pair
// ============================================================================
//
// Clusters of two CTAs.  Each CTA stages its own 128 rows of the activation
// tile and its own BN/2 rows of the weight tile, so a pair reads 256 + BN
// operand rows per K slice for a 256 x BN output tile: per SM that is half the
// weight rows of gemm_tile_kernel's 128 x BN tile for the same MMA work.  The
// even CTA's MMA warp issues tcgen05.mma.cta_group::2 (M = 256); each CTA's
// TMEM holds its own 128 accumulator rows, and each CTA's epilogue warps
// finish their own rows exactly as in gemm_tile_kernel.
//
// Barriers: the stage-full barriers of the even CTA count the transaction
// bytes of both CTAs' loads (each CTA's loads complete on them through
// cta_group::2 TMA); the MMA's commits arrive on the stage-empty and
// accumulator-full barriers of both CTAs; the accumulator-empty barriers of
// the even CTA take one arrival from each epilogue warp of both CTAs.
template <int BN, bool MIXED = false>
struct PairCfg {
    static constexpr int A_BYTES = kBM * kBKB;            // this CTA's 128 activation rows
    static constexpr int B_BYTES = (BN / 2) * kBKB;       // this CTA's BN/2 weight rows
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int STAGES_RAW = kSmemBudget / STAGE;
    static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
    static constexpr int BUF_COLS = MIXED ? 2 * BN : BN;  // int32 acc (+ fp32 outlier acc)
    static constexpr int TMEM_COLS = 2 * BUF_COLS <= 256 ? 256 : 512;
    static_assert(2 * BUF_COLS <= 512, "TMEM holds 512 columns");
    static constexpr int SMEM = STAGES * STAGE + kEpiStageBytes + kEpiConstBytes + 1024;
    static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "BN");
    static_assert((BN / 2) % 8 == 0, "weight half-tile rows: whole 8-row swizzle atoms");
};

template <int BN, int KIND, bool QOUT, bool GROUPED = false, bool MIXED = false>
__global__ void __launch_bounds__(kThreads, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmA16, const __grid_constant__ CUtensorMap tmB16,
                 const __grid_constant__ CUtensorMap tmY, int use_tmy, const EpiParams p, int num_kb,
                 int tiles_m, int tiles_n, const int32_t* group_offsets, int experts) {
    using C = PairCfg<BN, MIXED>;
    static_assert(!(GROUPED && MIXED), "grouped tiles carry no outlier stream");
    __shared__ int g_off[GROUPED ? kMaxGroupedExperts + 1 : 1];
    __shared__ int g_mt[GROUPED ? kMaxGroupedExperts + 1 : 1];
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    __shared__ __align__(8) uint64_t full_bar[C::STAGES];
    __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint32_t rank = cluster_ctarank();          // 0: issues the pair's MMAs
    const int pair = static_cast<int>(blockIdx.x >> 1);
    const int npairs = static_cast<int>(gridDim.x >> 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull_bar[b], 1);
            mbar_init(&tempty_bar[b], 8);   // 4 epilogue warps x 2 CTAs
        }
        mbar_init(&drain_bar, 1);
        abort_sh = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(&tmem_base_sh, C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    if constexpr (GROUPED) {
        // The routing offsets come from the previous kernels.
        pdl_wait();
        if (warp == 2) build_group_map(group_offsets, experts, p.m, 2 * kBM, g_off, g_mt);
    }
    tc_fence_before();
    __syncthreads();
    // Both CTAs' barriers are initialized before either touches the other's.
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;
    pdl_launch_dependents();

    const int num_tiles = GROUPED ? g_mt[GROUPED ? experts : 0] * tiles_n : tiles_m * tiles_n;
    // LLM.int8: the fp16 outlier K blocks (64 columns each) follow the int8
    // ones; their count is read on the device (no host round trip).
    int n16_kb = 0;
    if constexpr (MIXED) {
        // The producer reads the count after its early weight loads.
        if (warp != 0) {
            pdl_wait();
            n16_kb = (*p.outlier_count + 63) / 64;
        }
    }
    const int total_kb = num_kb + n16_kb;
    // A pair tile is 256 activation rows (128 from each CTA) x BN columns.
    auto tile_ref = [&](int tile) -> TileRef {
        if constexpr (GROUPED) return grouped_tile(tile, g_off, g_mt, experts, 2 * kBM, BN, p.n);
        else return dense_tile(tile, tiles_m, 2 * kBM, BN, p.m);
    };
    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (elect_one()) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            const uint32_t full0 = map_shared_rank(smem_addr(&full_bar[0]), 0);
            // The weights do not depend on the previous kernel: the first ring
            // of the first tile's weight halves goes out before the
            // programmatic-launch wait, the activation slices after it.
            int npre = 0;
            if constexpr (!GROUPED) {
                if (pair < num_tiles) {
                    const TileRef tr0 = tile_ref(pair);
                    const int yb0 = tr0.b_row + static_cast<int>(rank) * (BN / 2);
                    npre = num_kb < C::STAGES ? num_kb : C::STAGES;
                    for (int s = 0; s < npre; ++s) {
                        if (rank == 0) mbar_arrive_expect_tx(&full_bar[s], 2 * C::STAGE);
                        tma_load_2d_pair(smem + s * C::STAGE + C::A_BYTES, &tmB, full0 + 8u * static_cast<uint32_t>(s),
                                         s * kBKB, yb0);
                    }
                }
            }
            pdl_wait();
            int ptotal_kb = total_kb;
            if constexpr (MIXED) ptotal_kb = num_kb + (*p.outlier_count + 63) / 64;
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
                const TileRef tr = tile_ref(tile);
                for (int kb = 0; kb < ptotal_kb; ++kb) {
                    const bool pre = tile == pair && kb < npre;   // weight half already out
                    if (!pre && !mbar_wait(&empty_bar[stage], phase ^ 1, &abort_sh, p.status)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + stage * C::STAGE;
                    uint8_t* sb = sa + C::A_BYTES;
                    if (rank == 0 && !pre) mbar_arrive_expect_tx(&full_bar[stage], 2 * C::STAGE);
                    const uint32_t fb = full0 + 8u * static_cast<uint32_t>(stage);
                    const int ya = tr.a_row + static_cast<int>(rank) * kBM;
                    const int yb = tr.b_row + static_cast<int>(rank) * (BN / 2);
                    if (!MIXED || kb < num_kb) {
                        tma_load_2d_pair(sa, &tmA, fb, kb * kBKB, ya);
                        if (!pre) tma_load_2d_pair(sb, &tmB, fb, kb * kBKB, yb);
                    } else {
                        // 64 fp16 columns: the same 128-byte rows
                        tma_load_2d_pair(sa, &tmA16, fb, (kb - num_kb) * 64, ya);
                        tma_load_2d_pair(sb, &tmB16, fb, (kb - num_kb) * 64, yb);
                    }
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (even CTA)
        if (rank == 0 && elect_one()) {
            const uint32_t idesc = KIND == kE4M3 ? make_idesc(1, 0, 0, 2 * kBM, BN)
                                                 : make_idesc(2, 1, KIND == kS8U8 ? 0 : 1, 2 * kBM, BN);
            const uint32_t idesc16 = make_idesc(1, 0, 0, 2 * kBM, BN);   // f16 x f16 -> f32
            int stage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t bphase = 0;
            bool ok = true;
            for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
                if (!mbar_wait(&tempty_bar[buf], bphase ^ 1, &abort_sh, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + buf * C::BUF_COLS;
                for (int kb = 0; kb < total_kb; ++kb) {
                    if (!mbar_wait(&full_bar[stage], phase, &abort_sh, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_addr(smem + stage * C::STAGE);
                    const uint64_t ad = sdesc_kmajor_sw128(sa);
                    const uint64_t bd = sdesc_kmajor_sw128(sa + C::A_BYTES);
                    if (!MIXED || kb < num_kb) {
#pragma unroll
                        for (int ks = 0; ks < kBKB / 32; ++ks) {
                            if constexpr (KIND == kE4M3)
                                mma_issue_pair<kKindF8>(d, ad + 2 * ks, bd + 2 * ks, idesc, (kb | ks) != 0);
                            else
                                mma_issue_pair<kKindI8>(d, ad + 2 * ks, bd + 2 * ks, idesc, (kb | ks) != 0);
                        }
                    } else {
#pragma unroll
                        for (int ks = 0; ks < kBKB / 32; ++ks)
                            mma_issue_pair<kKindF16>(d + BN, ad + 2 * ks, bd + 2 * ks, idesc16,
                                                     ((kb - num_kb) | ks) != 0);
                    }
                    tc_commit_pair(&empty_bar[stage], 0x3);
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                tc_commit_pair(&tfull_bar[buf], 0x3);
                buf ^= 1;
                if (buf == 0) bphase ^= 1;
            }
            if (!ok) {
                // Abort: wait for the MMAs already issued before TMEM is freed.
                tc_commit_pair_local(&drain_bar);
                mbar_wait(&drain_bar, 0, nullptr, nullptr);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (both CTAs)
        pdl_wait();
        const int q = warp & 3;
        const uint32_t tempty0 = map_shared_rank(smem_addr(&tempty_bar[0]), 0);
        uint32_t sbuf = 0;
        uint8_t* epi_smem = smem + C::STAGES * C::STAGE;
        float* colc = reinterpret_cast<float*>(epi_smem + kEpiStageBytes) + (warp - 2) * 3 * BN;
        EpiStore es{use_tmy ? &tmY : nullptr, epi_smem + (warp - 2) * 4096, 0, &sbuf, colc, 0.f, 0, p.m,
                    false};
        const int rbase = static_cast<int>(rank) * kBM + q * 32 + lane;   // this thread's row in a tile
        EpiConsts<BN> pf;
        if (pair < num_tiles) {
            const TileRef t0 = tile_ref(pair);
            pf.fetch(p, t0.n_tile, t0.col_off, t0.a_row + rbase, t0.row_end);
        }
        int buf = 0;
        uint32_t bphase = 0;
        for (int tile = pair; tile < num_tiles; tile += npairs) {
            const TileRef tr = tile_ref(tile);
            if (!mbar_wait(&tfull_bar[buf], bphase, &abort_sh, p.status)) break;
            tc_fence_after();
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * C::BUF_COLS;
            es.row0 = tr.a_row + static_cast<int>(rank) * kBM + q * 32;
            es.row_end = tr.row_end;
            // A tensor store clips at the output's last row only: chunks that
            // cross an expert's end are stored row by row.
            es.tma_tile = GROUPED ? es.row0 + 32 <= tr.row_end : es.row0 < tr.row_end;
            pf.publish(colc);
            es.sx = pf.sx;
            es.rs = pf.rs;
            const int nt = tile + npairs;
            if (nt < num_tiles) {
                const TileRef tn = tile_ref(nt);
                pf.fetch(p, tn.n_tile, tn.col_off, tn.a_row + rbase, tn.row_end);
            }
            epilogue_tile<BN, KIND, MIXED, QOUT>(p, tb, es.row0 + lane, tr.n_tile, n16_kb, es);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty0 + 8u * static_cast<uint32_t>(buf));
            buf ^= 1;
            if (buf == 0) bphase ^= 1;
        }
        if (lane == 0) bulk_wait_all();   // staged output stores done before the CTA ends
        __syncwarp();
    }

    __syncthreads();
    // No CTA leaves while its partner may still signal one of its barriers or
    // read its shared memory.
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

// ============================================================================
// Decode kernel: weights as the MMA's M side, tokens as N, split-K in a cluster
// ============================================================================
template <int NT, int KIND>
struct DecodeCfg {
    static constexpr int A_BYTES = kBM * kBKB;   // 128 weight rows
    static constexpr int B_BYTES = NT * kBKB;    // NT token rows
    static constexpr int STAGE = A_BYTES + B_BYTES;
    // Partials pushed by every rank: [rank][tokens owned][128 channels], at most
    // 8 ranks each owning ceil(NT / ranks) tokens.
    static constexpr int RED_BYTES = (NT + 8) * kBM * 4;
    static constexpr int STAGES_RAW = (kSmemBudget - RED_BYTES) / STAGE;
    static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
    static constexpr int TMEM_COLS = NT < 32 ? 32 : NT;
    static constexpr int SMEM = STAGES * STAGE + RED_BYTES + 1024;
};

template <int NT, int KIND, bool QOUT>
__global__ void __launch_bounds__(kThreads, 1)
gemm_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                   const EpiParams p, int num_kb, int kb_per_split, int splits, int nstages) {
    using C = DecodeCfg<NT, KIND>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint32_t* red = reinterpret_cast<uint32_t*>(smem + nstages * C::STAGE);  // [NT][128]
    __shared__ __align__(8) uint64_t full_bar[C::STAGES];
    __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
    __shared__ __align__(8) uint64_t tfull_bar;
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;
    __shared__ float sx_sh[NT];       // token scales and row sums, loaded while the MMAs run
    __shared__ int32_t rowsum_sh[NT];

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int tn = blockIdx.x;                       // 128 output channels
    const uint32_t rank = cluster_ctarank();         // split index along K
    const int kb0 = static_cast<int>(rank) * kb_per_split;
    const int kb1 = min(num_kb, kb0 + kb_per_split);
    const int my_kb = kb1 > kb0 ? kb1 - kb0 : 0;
    // Epilogue constants of this thread's output channel (epilogue warps).
    float e_sw = 0.f, e_zw = 0.f, e_bias = 0.f;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nstages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&tfull_bar, 1);
        mbar_init(&drain_bar, 1);
        abort_sh = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;
    // The next kernel (typically the next layer's activation quantizer, which
    // waits for this grid before touching memory) may launch now.
    pdl_launch_dependents();

    if (warp == 0) {
        if (elect_one()) {
            tma_prefetch_desc(&tmW);
            tma_prefetch_desc(&tmX);
            // The weights do not depend on the previous kernel: their first
            // ring of loads goes out before the programmatic-launch wait, the
            // activation codes of the same stages right after it.
            const int first = my_kb < nstages ? my_kb : nstages;
            for (int i = 0; i < first; ++i) {
                uint8_t* sa = smem + i * C::STAGE;
                mbar_arrive_expect_tx(&full_bar[i], C::STAGE);
                tma_load_2d(sa, &tmW, &full_bar[i], (kb0 + i) * kBKB, tn * kBM);
            }
            pdl_wait();
            for (int i = 0; i < first; ++i)
                tma_load_2d(smem + i * C::STAGE + C::A_BYTES, &tmX, &full_bar[i], (kb0 + i) * kBKB, 0);
            uint32_t issued = (1u << first) - 1u, last_par = 0;
            int stage = first == nstages ? 0 : first;
            uint32_t phase = first == nstages ? 1u : 0u;
            bool ok = true;
            for (int kb = kb0 + first; kb < kb1; ++kb) {
                if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_sh, p.status)) {
                    ok = false;
                    break;
                }
                uint8_t* sa = smem + stage * C::STAGE;
                mbar_arrive_expect_tx(&full_bar[stage], C::STAGE);
                tma_load_2d(sa, &tmW, &full_bar[stage], kb * kBKB, tn * kBM);
                tma_load_2d(sa + C::A_BYTES, &tmX, &full_bar[stage], kb * kBKB, 0);
                issued |= 1u << stage;
                last_par = (last_par & ~(1u << stage)) | (phase << stage);
                if (++stage == nstages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            if (!ok)
                for (int s = 0; s < nstages; ++s)
                    if (issued & (1u << s)) mbar_wait(&full_bar[s], (last_par >> s) & 1, nullptr, nullptr);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (elect_one()) {
            // A = weights (u8 or s8 for INT8, E4M3), B = tokens.
            const uint32_t idesc = KIND == kE4M3 ? make_idesc(1, 0, 0, kBM, NT)
                                                 : make_idesc(2, KIND == kS8U8 ? 0 : 1, 1, kBM, NT);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int i = 0; i < my_kb; ++i) {
                if (!mbar_wait(&full_bar[stage], phase, &abort_sh, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = smem_addr(smem + stage * C::STAGE);
                const uint64_t ad = sdesc_kmajor_sw128(sa);
                const uint64_t bd = sdesc_kmajor_sw128(sa + C::A_BYTES);
#pragma unroll
                for (int ks = 0; ks < kBKB / 32; ++ks) {
                    if constexpr (KIND == kE4M3)
                        mma_issue<kKindF8>(tmem_base, ad + 2 * ks, bd + 2 * ks, idesc, (i | ks) != 0);
                    else
                        mma_issue<kKindI8>(tmem_base, ad + 2 * ks, bd + 2 * ks, idesc, (i | ks) != 0);
                }
                tc_commit(&empty_bar[stage]);
                if (++stage == nstages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            tc_commit(ok ? &tfull_bar : &drain_bar);
            if (!ok) mbar_wait(&drain_bar, 0, nullptr, nullptr);
        }
        __syncwarp();
    } else {
        // Epilogue warps: push this rank's TMEM partial for token t into the
        // shared memory of the rank that finishes t (t % splits), at slot
        // [rank][t / splits][channel].
        const int q = warp & 3;
        const int ch = q * 32 + lane;
        const int tpo = (NT + splits - 1) / splits;     // tokens owned per rank
        // The dequant inputs go out now, not after the reduction: the weight
        // scales and zero points do not depend on the previous kernel, the
        // token scales and row sums (its outputs) are complete after the wait.
        {
            const int n = tn * kBM + ch;
            if (n < p.n) {
                e_sw = p.sw[n];
                if (p.zw) e_zw = p.zw[n];
                if (p.bias) e_bias = p.bias[n];
            }
            pdl_wait();
            const int t = q * 32 + lane;
            if (t < NT) {
                sx_sh[t] = t < p.m ? p.sx[t] : 0.f;
                rowsum_sh[t] = (t < p.m && p.zw) ? p.rowsum[t] : 0;
            }
        }
        bool have = my_kb > 0 && mbar_wait(&tfull_bar, 0, &abort_sh, p.status);
        if (have) tc_fence_after();
        __syncwarp();
        const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
        const uint32_t red_base = smem_addr(red);
#pragma unroll
        for (int c = 0; c < NT; c += 16) {
            uint32_t r[16];
            tmem_ld16(tb + c, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int t = c + i;
                const uint32_t owner = static_cast<uint32_t>(t % splits);
                const uint32_t off = ((rank * tpo + t / splits) * kBM + ch) * 4u;
                st_shared_cluster_u32(map_shared_rank(red_base + off, owner), have ? r[i] : 0u);
            }
        }
        __syncwarp();
    }

    // Every rank's pushed partials are visible after this barrier; after it no
    // CTA touches another CTA's shared memory, so each may exit when done.
    __syncthreads();
    cluster_sync();

    if (warp >= 2) {
        // Rank r finishes the tokens t with t % splits == r, summing the
        // partials in rank order.
        const int q = warp & 3;
        const int ch = q * 32 + lane;
        const int tpo = (NT + splits - 1) / splits;
        const int n = tn * kBM + ch;
        const bool has_zp = p.zw != nullptr;
        const bool col_ok = n < p.n;
        const float sw = e_sw, zw = e_zw, bias = e_bias;
        for (int t = static_cast<int>(rank); t < NT && t < p.m; t += splits) {
            const int tl = t / splits;
            uint32_t acc_bits;
            float v;
            if constexpr (KIND == kE4M3) {
                float s = 0.f;
                for (int r = 0; r < splits; ++r)
                    s = __fadd_rn(s, __uint_as_float(red[(r * tpo + tl) * kBM + ch]));
                acc_bits = __float_as_uint(s);
                v = __fmul_rn(__fmul_rn(s, sx_sh[t]), sw);
            } else {
                int32_t s = 0;
                for (int r = 0; r < splits; ++r)
                    s += static_cast<int32_t>(red[(r * tpo + tl) * kBM + ch]);
                acc_bits = static_cast<uint32_t>(s);
                v = dequant_int(s, zw, rowsum_sh[t], sx_sh[t], sw, has_zp);
            }
            if (p.bias) v = __fadd_rn(v, bias);
            if (col_ok) {
                if constexpr (QOUT)
                    p.yq[static_cast<int64_t>(t) * p.ldy + n] = static_cast<int8_t>(requant_code_fast(v, requant_consts(p.out_scale)));
                else
                    p.y[static_cast<int64_t>(t) * p.ldy + n] = __float2bfloat16_rn(v);
                if (p.acc_debug)
                    static_cast<uint32_t*>(p.acc_debug)[static_cast<int64_t>(t) * p.n + n] = acc_bits;
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}


// ============================================================================
// Host side
// ============================================================================
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

// 2-D K-major tile map with 128-byte swizzle: inner extent `inner` elements of
// `esize` bytes, `outer` rows `ld_bytes` apart, box of (box_inner, box_outer).
bool make_map(CUtensorMap* m, const void* base, bool fp16, uint64_t inner, uint64_t outer,
              uint64_t ld_bytes, uint32_t box_inner, uint32_t box_outer) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {ld_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map of the bf16 output for the epilogue's staged stores: boxes of
// 32 columns x 32 rows with the 64-byte swizzle of the staging buffers.
bool make_map_y(CUtensorMap* m, const void* y, uint64_t n, uint64_t rows, uint64_t ldy_elems) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {n, rows};
    const cuuint64_t strides[1] = {ldy_elems * 2};
    const cuuint32_t box[2] = {32, 32};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(y), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
    static int cached[64] = {0};
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return n;
    }
    if (cached[dev] > 0) return cached[dev];
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return 148;
    }
    cached[dev] = n;
    return n;
}

// The dynamic shared-memory limit is a per-kernel, per-device attribute: it is
// set once (to the largest size asked for) instead of on every launch, which
// keeps the host side of a call short.
template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
    static std::mutex mu;
    static std::unordered_map<const void*, int> done[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    }
    const void* key = reinterpret_cast<const void*>(kernel);
    {
        std::lock_guard<std::mutex> lk(mu);
        auto it = done[dev].find(key);
        if (it != done[dev].end() && it->second >= bytes) return cudaSuccess;
    }
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) {
        std::lock_guard<std::mutex> lk(mu);
        int& v = done[dev][key];
        if (bytes > v) v = bytes;
    }
    return e;
}

template <int BN, int KIND, bool MIXED, bool QOUT = false>
q8_status run_tile(const LinearArgs& a, const EpiParams& ep, cudaStream_t s) {
    using C = TileCfg<BN, MIXED>;
    CUtensorMap tA, tB, tA16, tB16;
    if (!make_map(&tA, a.a_codes, false, a.k, a.m, a.lda, kBKB, kBM) ||
        !make_map(&tB, a.b_codes, false, a.k, a.n, a.ldb, kBKB, BN))
        return Q8_ERR_CUDA;
    if constexpr (MIXED) {
        if (!make_map(&tA16, a.xo, true, a.k16_cap, a.m, a.ldxo * 2, 64, kBM) ||
            !make_map(&tB16, a.wo, true, a.k16_cap, a.n, a.ldwo * 2, 64, BN))
            return Q8_ERR_CUDA;
    } else {
        tA16 = tA;
        tB16 = tB;
    }
    CUtensorMap tY = tA;
    const int use_tmy = (!QOUT && a.y != nullptr && make_map_y(&tY, a.y, a.n, a.m, a.ldy)) ? 1 : 0;
    auto kern = gemm_tile_kernel<BN, KIND, MIXED, QOUT>;
    if (set_smem(kern, C::SMEM) != cudaSuccess) return Q8_ERR_LAUNCH;
    const int tiles_m = static_cast<int>((a.m + kBM - 1) / kBM);
    const int tiles_n = static_cast<int>((a.n + BN - 1) / BN);
    const int tiles = tiles_m * tiles_n;
    const int num_kb = static_cast<int>((a.k + kBKB - 1) / kBKB);
    const int grid = tiles < sm_count() ? tiles : sm_count();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tA, tB, tA16, tB16, tY, use_tmy, ep, num_kb, tiles_m, tiles_n,
                           static_cast<const int32_t*>(nullptr), 0) != cudaSuccess) {
        cudaGetLastError();
        return Q8_ERR_LAUNCH;
    }
    return Q8_OK;
}

// Pairs that fit on the device at once (clusters of two 1-CTA-per-SM CTAs),
// cached per kernel instantiation and device.
template <typename K>
int max_pairs(K kernel, int smem) {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return sm_count() / 2;
    if (cached[dev] > 0) return cached[dev];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = sm_count() / 2;
    }
    cached[dev] = n;
    return n;
}

template <int BN, int KIND, bool QOUT = false, bool MIXED = false>
q8_status run_pair(const LinearArgs& a, const EpiParams& ep, cudaStream_t s) {
    using C = PairCfg<BN, MIXED>;
    CUtensorMap tA, tB, tA16, tB16;
    if (!make_map(&tA, a.a_codes, false, a.k, a.m, a.lda, kBKB, kBM) ||
        !make_map(&tB, a.b_codes, false, a.k, a.n, a.ldb, kBKB, BN / 2))
        return Q8_ERR_CUDA;
    if constexpr (MIXED) {
        if (!make_map(&tA16, a.xo, true, a.k16_cap, a.m, a.ldxo * 2, 64, kBM) ||
            !make_map(&tB16, a.wo, true, a.k16_cap, a.n, a.ldwo * 2, 64, BN / 2))
            return Q8_ERR_CUDA;
    } else {
        tA16 = tA;
        tB16 = tB;
    }
    CUtensorMap tY = tA;
    const int use_tmy = (!QOUT && a.y != nullptr && make_map_y(&tY, a.y, a.n, a.m, a.ldy)) ? 1 : 0;
    auto kern = gemm_pair_kernel<BN, KIND, QOUT, false, MIXED>;
    if (set_smem(kern, C::SMEM) != cudaSuccess) return Q8_ERR_LAUNCH;
    const int tiles_m = static_cast<int>((a.m + 2 * kBM - 1) / (2 * kBM));
    const int tiles_n = static_cast<int>((a.n + BN - 1) / BN);
    const int tiles = tiles_m * tiles_n;
    const int num_kb = static_cast<int>((a.k + kBKB - 1) / kBKB);
    const int pairs_max = max_pairs(kern, C::SMEM);
    const int pairs = tiles < pairs_max ? tiles : pairs_max;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kern, tA, tB, tA16, tB16, tY, use_tmy, ep, num_kb, tiles_m, tiles_n,
                           static_cast<const int32_t*>(nullptr), 0) != cudaSuccess) {
        cudaGetLastError();
        return Q8_ERR_LAUNCH;
    }
    return Q8_OK;
}

template <int NT, int KIND, bool QOUT = false>
q8_status run_decode(const LinearArgs& a, const EpiParams& ep, cudaStream_t s) {
    using C = DecodeCfg<NT, KIND>;
    CUtensorMap tW, tX;
    if (!make_map(&tW, a.b_codes, false, a.k, a.n, a.ldb, kBKB, kBM) ||
        !make_map(&tX, a.a_codes, false, a.k, a.m, a.lda, kBKB, NT))
        return Q8_ERR_CUDA;
    auto kern = gemm_decode_kernel<NT, KIND, QOUT>;
    if (set_smem(kern, C::SMEM) != cudaSuccess) return Q8_ERR_LAUNCH;
    const int tiles_n = static_cast<int>((a.n + kBM - 1) / kBM);
    const int num_kb = static_cast<int>((a.k + kBKB - 1) / kBKB);
    // Split K across the CTAs of a cluster (at most 8, every split non-empty)
    // so that the grid fills the SMs at two CTAs per SM, which the short stage
    // ring of a split allows.
    int want = 2 * sm_count() / tiles_n;
    if (want < 1) want = 1;
    if (want > 8) want = 8;
    if (want > num_kb) want = num_kb;
    const int per = (num_kb + want - 1) / want;
    const int splits = (num_kb + per - 1) / per;
    const int nstages = per < C::STAGES ? per : C::STAGES;
    const int smem = nstages * C::STAGE + C::RED_BYTES + 1024;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles_n), static_cast<unsigned>(splits), 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = static_cast<unsigned>(splits);
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kern, tW, tX, ep, num_kb, per, splits, nstages) != cudaSuccess) {
        cudaGetLastError();
        return Q8_ERR_LAUNCH;
    }
    return Q8_OK;
}


template <int BN>
q8_status run_grouped(const MoeArgs& a, const EpiParams& ep, cudaStream_t s) {
    using C = TileCfg<BN, false>;
    CUtensorMap tA, tB, tY;
    if (!make_map(&tA, a.x_codes, false, a.k, a.m, a.ldx, kBKB, kBM) ||
        !make_map(&tB, a.w_codes, false, a.k, a.experts * a.n, a.ldw, kBKB, BN))
        return Q8_ERR_CUDA;
    const int use_tmy = make_map_y(&tY, a.y, a.n, a.m, a.ldy) ? 1 : 0;
    if (!use_tmy) tY = tA;
    auto kern = gemm_tile_kernel<BN, kE4M3, false, false, true>;
    if (set_smem(kern, C::SMEM) != cudaSuccess) return Q8_ERR_LAUNCH;
    const int tiles_n = static_cast<int>((a.n + BN - 1) / BN);
    // Upper bound of the tiles (each expert adds at most one partial row tile);
    // the kernel reads the offsets and walks the actual ones.
    const int64_t upper = ((a.m + kBM - 1) / kBM + a.experts) * tiles_n;
    const int sms = sm_count();
    const int grid = static_cast<int>(upper < sms ? upper : sms);
    const int num_kb = static_cast<int>((a.k + kBKB - 1) / kBKB);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tA, tB, tA, tB, tY, use_tmy, ep, num_kb, 0, tiles_n, a.offsets,
                           static_cast<int>(a.experts)) != cudaSuccess) {
        cudaGetLastError();
        return Q8_ERR_LAUNCH;
    }
    return Q8_OK;
}

template <int KIND>
q8_status dispatch_kind(const LinearArgs& a, const EpiParams& ep, cudaStream_t s) {
    if constexpr (KIND != kE4M3) {
        if (a.yq != nullptr && a.m <= 64) {   // INT8 output codes
            if (a.m <= 16) return run_decode<16, KIND, true>(a, ep, s);
            if (a.m <= 32) return run_decode<32, KIND, true>(a, ep, s);
            return run_decode<64, KIND, true>(a, ep, s);
        }
    }
    if (a.m <= 16) return run_decode<16, KIND>(a, ep, s);
    if (a.m <= 32) return run_decode<32, KIND>(a, ep, s);
    if (a.m <= 64) return run_decode<64, KIND>(a, ep, s);
    if (a.m > 2 * kBM) {
        // 256-row tiles on CTA pairs.  Tile width: the persistent grid's
        // makespan is ceil(tiles / pairs) tiles of time proportional to BN,
        // so pick the BN with the smallest waves x BN (the wider on ties).
        const int64_t pairs = sm_count() / 2;
        const int cand[3] = {256, 224, 192};
        int best = 256;
        int64_t best_cost = INT64_MAX;
        for (int bn : cand) {
            const int64_t tiles = ((a.m + 255) / 256) * ((a.n + bn - 1) / bn);
            const int64_t cost = ((tiles + pairs - 1) / pairs) * bn;
            if (cost < best_cost) {
                best_cost = cost;
                best = bn;
            }
        }
        if constexpr (KIND != kE4M3) {
            if (a.yq != nullptr) {   // INT8 output codes
                if (best == 256) return run_pair<256, KIND, true>(a, ep, s);
                if (best == 224) return run_pair<224, KIND, true>(a, ep, s);
                return run_pair<192, KIND, true>(a, ep, s);
            }
        }
        if (best == 256) return run_pair<256, KIND>(a, ep, s);
        if (best == 224) return run_pair<224, KIND>(a, ep, s);
        return run_pair<192, KIND>(a, ep, s);
    }
    // Output tile width: the persistent grid's makespan is
    // ceil(tiles / SMs) tiles of time proportional to BN, so pick the BN with
    // the smallest waves x BN (the wider tile on ties).
    const int64_t sms = sm_count();
    const int cand[3] = {256, 224, 128};
    int best = 256;
    int64_t best_cost = INT64_MAX;
    for (int bn : cand) {
        const int64_t tiles = ((a.m + 127) / 128) * ((a.n + bn - 1) / bn);
        const int64_t cost = ((tiles + sms - 1) / sms) * bn;
        if (cost < best_cost) {
            best_cost = cost;
            best = bn;
        }
    }
    if constexpr (KIND != kE4M3) {
        if (a.yq != nullptr) {   // INT8 output codes
            if (best == 256) return run_tile<256, KIND, false, true>(a, ep, s);
            if (best == 224) return run_tile<224, KIND, false, true>(a, ep, s);
            return run_tile<128, KIND, false, true>(a, ep, s);
        }
    }
    if (best == 256) return run_tile<256, KIND, false>(a, ep, s);
    if (best == 224) return run_tile<224, KIND, false>(a, ep, s);
    return run_tile<128, KIND, false>(a, ep, s);
}

}  // namespace


template <int BN>
q8_status run_grouped_pair(const MoeArgs& a, const EpiParams& ep, cudaStream_t s) {
    using C = PairCfg<BN>;
    CUtensorMap tA, tB, tY;
    if (!make_map(&tA, a.x_codes, false, a.k, a.m, a.ldx, kBKB, kBM) ||
        !make_map(&tB, a.w_codes, false, a.k, a.experts * a.n, a.ldw, kBKB, BN / 2))
        return Q8_ERR_CUDA;
    const int use_tmy = make_map_y(&tY, a.y, a.n, a.m, a.ldy) ? 1 : 0;
    if (!use_tmy) tY = tA;
    auto kern = gemm_pair_kernel<BN, kE4M3, false, true>;
    if (set_smem(kern, C::SMEM) != cudaSuccess) return Q8_ERR_LAUNCH;
    const int tiles_n = static_cast<int>((a.n + BN - 1) / BN);
    const int64_t upper = ((a.m + 2 * kBM - 1) / (2 * kBM) + a.experts) * tiles_n;
    const int pairs_max = max_pairs(kern, C::SMEM);
    const int pairs = static_cast<int>(upper < pairs_max ? upper : pairs_max);
    const int num_kb = static_cast<int>((a.k + kBKB - 1) / kBKB);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kern, tA, tB, tA, tB, tY, use_tmy, ep, num_kb, 0, tiles_n, a.offsets,
                           static_cast<int>(a.experts)) != cudaSuccess) {
        cudaGetLastError();
        return Q8_ERR_LAUNCH;
    }
    return Q8_OK;
}

// Grouped FP8 rowwise linear on the persistent kernels with the expert-aware
// tile map (at most kMaxGroupedExperts experts); Q8_ERR_SHAPE tells the
// caller to use the one-tile-per-CTA kernel instead.
q8_status launch_grouped_fp8(const MoeArgs& a, cudaStream_t s) {
    if (a.experts > kMaxGroupedExperts) return Q8_ERR_SHAPE;
    if (a.m == 0 || a.n == 0) return Q8_OK;
    EpiParams ep = {};
    ep.m = static_cast<int>(a.m);
    ep.n = static_cast<int>(a.n);
    ep.sx = a.sx;
    ep.sw = a.sw;
    ep.bias = a.bias;
    ep.y = a.y;
    ep.ldy = a.ldy;
    ep.status = device_status_ptr();
    // With 256 or more tokens per expert on average, 256-row tiles on CTA
    // pairs: half the operand traffic per SM of 128-row tiles, which is what
    // bounds these GEMMs, for at most half a tile of padding per expert.
    if (a.m >= 256 * a.experts) {
        if (a.n % 256 == 0 || a.n > 2048) return run_grouped_pair<256>(a, ep, s);
        return run_grouped_pair<128>(a, ep, s);
    }
    // Output tile width: the persistent grid's makespan, waves x (BN + a
    // tile's fixed cost of about 64 columns' worth), over an estimate of the
    // row tiles (each expert adds about half a partial tile).
    const int64_t sms = sm_count();
    const int64_t rows_est = (a.m + kBM - 1) / kBM + a.experts / 2;
    const int cand[4] = {256, 224, 192, 128};
    int best = 256;
    int64_t best_cost = INT64_MAX;
    for (int bn : cand) {
        const int64_t tiles = rows_est * ((a.n + bn - 1) / bn);
        const int64_t cost = ((tiles + sms - 1) / sms) * (bn + 64);
        if (cost < best_cost) {
            best_cost = cost;
            best = bn;
        }
    }
    if (best == 256) return run_grouped<256>(a, ep, s);
    if (best == 224) return run_grouped<224>(a, ep, s);
    if (best == 192) return run_grouped<192>(a, ep, s);
    return run_grouped<128>(a, ep, s);
}

q8_status launch_linear(const LinearArgs& a, cudaStream_t s) {
    if (a.m == 0 || a.n == 0) return Q8_OK;
    EpiParams ep;
    ep.m = static_cast<int>(a.m);
    ep.n = static_cast<int>(a.n);
    ep.sx = a.sx;
    ep.rowsum = a.rowsum;
    ep.sw = a.sw;
    ep.zw = a.zw;
    ep.bias = a.bias;
    ep.y = a.y;
    ep.ldy = a.ldy;
    ep.yq = a.yq;
    ep.out_scale = a.out_scale;
    ep.acc_debug = a.acc_debug;
    ep.y16_debug = a.y16_debug;
    ep.outlier_count = a.outlier_count;
    ep.status = device_status_ptr();
    if (a.outlier_count != nullptr) {
        // More than one 128-row tile of tokens: 256-row tiles on CTA pairs
        // (a quarter fewer operand bytes per SM, which bounds these GEMMs).
        if (a.m > kBM) {
            if (a.kind == kS8U8) return run_pair<128, kS8U8, false, true>(a, ep, s);
            return run_pair<128, kS8S8, false, true>(a, ep, s);
        }
        if (a.kind == kS8U8) return run_tile<128, kS8U8, true>(a, ep, s);
        return run_tile<128, kS8S8, true>(a, ep, s);
    }
    switch (a.kind) {
        case kS8S8: return dispatch_kind<kS8S8>(a, ep, s);
        case kS8U8: return dispatch_kind<kS8U8>(a, ep, s);
        case kE4M3: return dispatch_kind<kE4M3>(a, ep, s);
    }
    return Q8_ERR_DTYPE;
}

}  // namespace q8
