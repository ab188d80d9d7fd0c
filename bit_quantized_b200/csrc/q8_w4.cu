// Group-wise 4-bit weights with 16-bit activations (W4A16) on the sm_100a
// tensor cores.
//
// What is computed (quantization overview "大模型量化技术", 2.2 granularity
// table: one scale per group of consecutive parameters; "大模型量化" (Xilyfe),
// GGUF section: absmax per block, qmax = 2^(4-1) - 1 = 7):
//   weights  S[j, r] = fl32(max |w| over group j of row r / 7), eps floor 1e-8
//            q = clamp(rne(fl32(w / S)), -7, 7), stored as the nibble q + 8
//   linear   w~ = round16(fl32(S q)) in the activation's 16-bit format,
//            y = sum_k x w~ (fp32 in TMEM), y = fl32(y + bias[n]), Y = bf16(y)
//
// Q4_K ("大模型量化" (Xilyfe), GGUF section, Q4_K simulation): groups of 32
// whose scales are quantized again per super block of 8, s_super = max / 15,
// 4-bit sub-scale codes; the kernel multiplies with fl32(s_super * code).
//
// Storage: codes are n x k/2 bytes, element 2j in the low nibble of byte j and
// element 2j+1 in the high nibble; scales are group-major, scale[j * n + r], so
// the 128 rows of a tile read one contiguous 512-byte run per group.
//
// w4a16_kernel: a CTA owns 128 output channels (the MMA's M side, one TMEM
// lane each) and NT tokens (the MMA's N side).  For small token counts the K
// range is split across the CTAs of a cluster and the fp32 partials are summed
// through distributed shared memory in rank order, as in the int8 decode GEMM.
//   warp 0     one lane streams, per 64-deep K slice, the packed codes and
//              scales (no swizzle) and the activation tile (128-byte swizzle)
//              into one slot of a staging ring by TMA; the first ring of codes
//              and scales goes out before the programmatic-launch wait;
//   warp 1     TMEM allocation; one lane issues tcgen05.mma kind::f16 with the
//              dequantized weight slice as A and the staged activation tile
//              as B, then frees both rings' slots;
//   warps 2-5  dequantize: thread r expands row r's 64 codes of a slice into
//              16-bit values written directly in the 128-byte-swizzled K-major
//              layout the MMA reads (a separate, shorter ring); then the same
//              warps run the epilogue.
// No TMA multicast is used.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "q8_device.cuh"
#include "q8_internal.h"

namespace q8 {
namespace {

constexpr float kEps = 1e-8f;

// ============================================================================
// Weight quantizer: one thread per group
// ============================================================================
__device__ __forceinline__ float widen1(__half h) { return __half2float(h); }
__device__ __forceinline__ float widen1(__nv_bfloat16 h) { return __bfloat162float(h); }

template <typename T>
__device__ __forceinline__ void widen8(const uint4& v, float (&f)[8]) {
    const T* h = reinterpret_cast<const T*>(&v);
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = widen1(h[i]);
}

template <typename T>
__global__ void __launch_bounds__(256)
group_quant_kernel(const T* __restrict__ W, int64_t n, int64_t k, int64_t ldw, int g,
                   uint8_t* __restrict__ codes, int64_t ldc, float* __restrict__ scale) {
    const int64_t ng = k / g;
    const int64_t id = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (id >= n * ng) return;
    const int64_t row = id / ng, grp = id % ng;
    const T* w = W + row * ldw + grp * g;
    float a = 0.f;
    for (int j = 0; j < g; j += 8) {
        float f[8];
        widen8<T>(*reinterpret_cast<const uint4*>(w + j), f);
#pragma unroll
        for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(f[i]));
    }
    float S = __fdiv_rn(a, 7.0f);
    if (!(S >= kEps)) S = kEps;
    uint8_t* out = codes + row * ldc + grp * (g / 2);
    for (int j = 0; j < g; j += 32) {
        uint32_t word[4];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            float f[8];
            widen8<T>(*reinterpret_cast<const uint4*>(w + j + 8 * v), f);
            uint32_t packed = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                int q = __float2int_rn(__fdiv_rn(f[i], S));
                q = q < -7 ? -7 : (q > 7 ? 7 : q);
                packed |= static_cast<uint32_t>(q + 8) << (4 * i);
            }
            word[v] = packed;
        }
        *reinterpret_cast<uint4*>(out + j / 2) = make_uint4(word[0], word[1], word[2], word[3]);
    }
    scale[grp * n + row] = S;
}

// ============================================================================
// Q4_K two-level scales: one thread per super block of 8 x 32 weights
// ============================================================================
// Sub-blocks are quantized exactly as groups of 32 above (codes from the
// unquantized sub-block scale); then s_super = fl32(max s_sub / 15) and the
// sub-block scale codes are clamp(rne(fl32(s_sub / s_super)), 0, 15).  The
// effective scale fl32(s_super * code) goes to the group-major scale array the
// W4A16 kernel reads; the compact form (two sub-scale codes per byte, low
// nibble = even sub-block, and the fp32 s_super) is written for storage.
template <typename T>
__global__ void __launch_bounds__(256)
q4k_quant_kernel(const T* __restrict__ W, int64_t n, int64_t k, int64_t ldw,
                 uint8_t* __restrict__ codes, int64_t ldc, float* __restrict__ scale,
                 uint8_t* __restrict__ sub_codes, float* __restrict__ super_scale) {
    const int64_t nb = k / 256;
    const int64_t id = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (id >= n * nb) return;
    const int64_t row = id / nb, blk = id % nb;
    float ss[8];
#pragma unroll 1
    for (int j = 0; j < 8; ++j) {
        const T* w = W + row * ldw + blk * 256 + j * 32;
        float f[4][8];
        float a = 0.f;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            widen8<T>(*reinterpret_cast<const uint4*>(w + 8 * v), f[v]);
#pragma unroll
            for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(f[v][i]));
        }
        float S = __fdiv_rn(a, 7.0f);
        if (!(S >= kEps)) S = kEps;
        uint32_t word[4];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            uint32_t packed = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                int q = __float2int_rn(__fdiv_rn(f[v][i], S));
                q = q < -7 ? -7 : (q > 7 ? 7 : q);
                packed |= static_cast<uint32_t>(q + 8) << (4 * i);
            }
            word[v] = packed;
        }
        *reinterpret_cast<uint4*>(codes + row * ldc + blk * 128 + j * 16) =
            make_uint4(word[0], word[1], word[2], word[3]);
        ss[j] = S;
    }
    float mx = ss[0];
#pragma unroll
    for (int j = 1; j < 8; ++j) mx = ss[j] > mx ? ss[j] : mx;
    const float sup = __fdiv_rn(mx, 15.0f);
    super_scale[blk * n + row] = sup;
    uint32_t pk = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        int c = __float2int_rn(__fdiv_rn(ss[j], sup));
        c = c < 0 ? 0 : (c > 15 ? 15 : c);
        scale[(blk * 8 + j) * n + row] = __fmul_rn(sup, static_cast<float>(c));
        pk |= static_cast<uint32_t>(c) << (4 * j);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
        sub_codes[(blk * 4 + j) * n + row] = static_cast<uint8_t>(pk >> (8 * j));
}

// scale[j * n + r] = fl32(s_super[(j / 8) * n + r] * code_j), code_j from the
// compact sub-scale codes.
__global__ void __launch_bounds__(256)
q4k_expand_kernel(const uint8_t* __restrict__ sub_codes, const float* __restrict__ super_scale,
                  int64_t n, int64_t k, float* __restrict__ scale) {
    const int64_t total = n * (k / 32);
    const int64_t id = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (id >= total) return;
    const int64_t j = id / n, r = id % n;
    const uint32_t c = (sub_codes[(j / 2) * n + r] >> (4 * (j & 1))) & 15u;
    scale[id] = __fmul_rn(super_scale[(j / 8) * n + r], static_cast<float>(c));
}

// ============================================================================
// W4A16 GEMM
// ============================================================================
constexpr int kDqWarps = 8;                     // dequantizing warps (2 .. 9)
constexpr int kThreads = 64 + 32 * kDqWarps;
constexpr int kBM = 128;                        // weight rows per CTA (MMA M)
constexpr int kBK = 64;                         // K elements per stage (128 bytes of 16-bit)
constexpr int kABytes = kBM * kBK * 2;          // 16 KB dequantized weight slice
constexpr int kQBytes = kBM * kBK / 2;          // 4 KB packed codes
constexpr int kSBytes = 2 * kBM * 4;            // room for two groups of scales
constexpr int kMaxA = 8;
constexpr int kMaxQ = 8;

// Staging slot of one K slice: [activation tile, 128-byte swizzled][codes][scales].
template <int NT>
struct W4Cfg {
    static constexpr int X_BYTES = NT * kBK * 2;
    static constexpr int QSLOT = X_BYTES + kQBytes + kSBytes;
    static constexpr bool SPLIT = NT <= 64;     // K split across a cluster
    static constexpr int RED_BYTES = SPLIT ? (NT + 8) * kBM * 4 : 0;
    static constexpr int TMEM_COLS = NT < 32 ? 32 : NT;
    static_assert(QSLOT % 1024 == 0, "staging slots keep 1024-byte alignment");
};

struct W4Params {
    int m, n;
    const float* bias;
    __nv_bfloat16* y;
    int64_t ldy;
    int* status;
};

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack16x2(float lo, float hi) {
    if constexpr (BF16) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<const uint32_t*>(&v);
    } else {
        const __half2 v = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<const uint32_t*>(&v);
    }
}

__device__ __forceinline__ uint64_t pair(uint32_t lo, uint32_t hi) {
    uint64_t v;
    asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "r"(lo), "r"(hi));
    return v;
}

// Eight codes (one 32-bit word; byte e holds element 2e in its low nibble and
// 2e+1 in its high nibble) -> eight 16-bit values round16(fl32(s * q)),
// q = nibble - 8, packed in element order.  `s2` holds s twice.
//   The float with bits 0x4B0000nn is 2^23 + nn; subtracting 2^23 + 8 leaves q
//   exactly.  Both lanes of each f32x2 step round to nearest like the scalar
//   operations, so the products are fl32(s * q).
template <bool BF16>
__device__ __forceinline__ uint4 dequant8(uint32_t word, uint64_t s2) {
    const uint32_t lo = word & 0x0F0F0F0Fu;          // elements 0, 2, 4, 6
    const uint32_t hi = (word >> 4) & 0x0F0F0F0Fu;   // elements 1, 3, 5, 7
    const uint64_t magic = 0x4B0000084B000008ull;    // {2^23 + 8, 2^23 + 8}
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const uint32_t sel = 0x7540u | static_cast<uint32_t>(e);   // byte e, 0, 0, 0x4B
        const uint64_t v = pair(__byte_perm(lo, 0x4B000000u, sel), __byte_perm(hi, 0x4B000000u, sel));
        uint64_t q, r;
        asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(q) : "l"(v), "l"(magic));
        asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(q), "l"(s2));
        uint32_t f0, f1;
        asm("mov.b64 {%0, %1}, %2;" : "=r"(f0), "=r"(f1) : "l"(r));
        o[e] = pack16x2<BF16>(__uint_as_float(f0), __uint_as_float(f1));
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

template <int NT, bool BF16>
__global__ void __launch_bounds__(kThreads, 2)
w4a16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmS,
             const __grid_constant__ CUtensorMap tmX, const W4Params p, int num_kb,
             int kb_per_split, int splits, int astages, int qstages, int group) {
    using C = W4Cfg<NT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* a_ring = smem;
    uint8_t* q_ring = a_ring + astages * kABytes;
    uint32_t* red = reinterpret_cast<uint32_t*>(q_ring + qstages * C::QSLOT);  // [rank][tok][128]

    __shared__ __align__(8) uint64_t q_full[kMaxQ];    // codes + scales landed
    __shared__ __align__(8) uint64_t x_full[kMaxQ];    // activation tile landed
    __shared__ __align__(8) uint64_t q_empty[kMaxQ];   // slot consumed by the MMAs
    __shared__ __align__(8) uint64_t a_full[kMaxA];    // 16-bit weight slice written
    __shared__ __align__(8) uint64_t a_empty[kMaxA];   // weight slice consumed
    __shared__ __align__(8) uint64_t tfull_bar;
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int tn = blockIdx.x;                                  // 128 output channels
    const int m0 = static_cast<int>(blockIdx.z) * NT;           // first token of the tile
    const uint32_t rank = splits > 1 ? cluster_ctarank() : 0u;  // split index along K
    const int kb0 = static_cast<int>(rank) * kb_per_split;
    const int kb1 = min(num_kb, kb0 + kb_per_split);
    const int my_kb = kb1 > kb0 ? kb1 - kb0 : 0;
    const int gps = group < kBK ? kBK / group : 1;             // scale groups per stage
    const uint32_t qs_tx = kQBytes + gps * kBM * 4;

    if (threadIdx.x == 0) {
        for (int s = 0; s < qstages; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&x_full[s], 1);
            mbar_init(&q_empty[s], 1);
        }
        for (int s = 0; s < astages; ++s) {
            mbar_init(&a_full[s], kDqWarps);   // one arrival per dequantizing warp
            mbar_init(&a_empty[s], 1);
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
    pdl_launch_dependents();

    if (warp == 0) {
        if (elect_one()) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmS);
            tma_prefetch_desc(&tmX);
            // Codes and scales do not depend on the previous kernel: the first
            // ring of them goes out before the programmatic-launch wait, the
            // activation tiles of the same slots right after it.
            const int first = my_kb < qstages ? my_kb : qstages;
            for (int i = 0; i < first; ++i) {
                uint8_t* dst = q_ring + i * C::QSLOT;
                mbar_arrive_expect_tx(&q_full[i], qs_tx);
                tma_load_2d(dst + C::X_BYTES, &tmQ, &q_full[i], (kb0 + i) * (kBK / 2), tn * kBM);
                tma_load_2d(dst + C::X_BYTES + kQBytes, &tmS, &q_full[i], tn * kBM,
                            ((kb0 + i) * kBK) / group);
            }
            pdl_wait();
            for (int i = 0; i < first; ++i) {
                mbar_arrive_expect_tx(&x_full[i], C::X_BYTES);
                tma_load_2d(q_ring + i * C::QSLOT, &tmX, &x_full[i], (kb0 + i) * kBK, m0);
            }
            uint32_t issued = (1u << first) - 1u, last_par = 0;
            int qs = first == qstages ? 0 : first;
            uint32_t qph = first == qstages ? 1u : 0u;
            bool ok = true;
            for (int kb = kb0 + first; kb < kb1; ++kb) {
                if (!mbar_wait(&q_empty[qs], qph ^ 1, &abort_sh, p.status)) {
                    ok = false;
                    break;
                }
                uint8_t* dst = q_ring + qs * C::QSLOT;
                mbar_arrive_expect_tx(&q_full[qs], qs_tx);
                tma_load_2d(dst + C::X_BYTES, &tmQ, &q_full[qs], kb * (kBK / 2), tn * kBM);
                tma_load_2d(dst + C::X_BYTES + kQBytes, &tmS, &q_full[qs], tn * kBM, (kb * kBK) / group);
                mbar_arrive_expect_tx(&x_full[qs], C::X_BYTES);
                tma_load_2d(dst, &tmX, &x_full[qs], kb * kBK, m0);
                issued |= 1u << qs;
                last_par = (last_par & ~(1u << qs)) | (qph << qs);
                if (++qs == qstages) {
                    qs = 0;
                    qph ^= 1;
                }
            }
            if (!ok)
                for (int s = 0; s < qstages; ++s)
                    if (issued & (1u << s)) {
                        mbar_wait(&q_full[s], (last_par >> s) & 1, nullptr, nullptr);
                        mbar_wait(&x_full[s], (last_par >> s) & 1, nullptr, nullptr);
                    }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (elect_one()) {
            const uint32_t idesc = make_idesc(1, BF16 ? 1 : 0, BF16 ? 1 : 0, kBM, NT);
            int as = 0, qs = 0;
            uint32_t aph = 0, qph = 0;
            bool ok = true;
            for (int i = 0; i < my_kb; ++i) {
                if (!mbar_wait(&a_full[as], aph, &abort_sh, p.status) ||
                    !mbar_wait(&x_full[qs], qph, &abort_sh, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t ad = sdesc_kmajor_sw128(smem_addr(a_ring + as * kABytes));
                const uint64_t bd = sdesc_kmajor_sw128(smem_addr(q_ring + qs * C::QSLOT));
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)   // four K = 16 steps of 32 bytes
                    mma_issue<kKindF16>(tmem_base, ad + 2 * ks, bd + 2 * ks, idesc, (i | ks) != 0);
                tc_commit(&a_empty[as]);
                tc_commit(&q_empty[qs]);
                if (++as == astages) {
                    as = 0;
                    aph ^= 1;
                }
                if (++qs == qstages) {
                    qs = 0;
                    qph ^= 1;
                }
            }
            tc_commit(ok ? &tfull_bar : &drain_bar);
            if (!ok) mbar_wait(&drain_bar, 0, nullptr, nullptr);
        }
        __syncwarp();
    } else {
        // ---------------- dequantize
        // Two threads per weight row, each expanding one half of the row's
        // 64-value slice (32 values: 16 bytes of codes, one scale group when
        // groups are 32 wide).  Neighbouring lanes read neighbouring 16-byte
        // code chunks (no bank conflicts), and the 8 lanes of a quarter warp
        // write 8 distinct swizzled chunks of 4 rows.
        const int ct = threadIdx.x - 64;
        const int row = ct >> 1, half = ct & 1;
        const uint32_t a_row = smem_addr(a_ring) + row * 128;
        const int sw = row & 7;
        int qs = 0, as = 0;
        uint32_t qph = 0, aph = 0;
        for (int i = 0; i < my_kb; ++i) {
            if (!mbar_wait(&q_full[qs], qph, &abort_sh, p.status)) break;
            const uint8_t* qsl = q_ring + qs * C::QSLOT + C::X_BYTES;
            const uint4 cw = *reinterpret_cast<const uint4*>(qsl + row * 32 + half * 16);
            const float* ssl = reinterpret_cast<const float*>(qsl + kQBytes);
            const uint32_t sc = __float_as_uint(ssl[(gps == 2 ? half * kBM : 0) + row]);
            if (!mbar_wait(&a_empty[as], aph ^ 1, &abort_sh, p.status)) break;
            const uint32_t dst = a_row + as * kABytes;
            const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
            const uint64_t s2 = pair(sc, sc);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint4 v = dequant8<BF16>(w[c], s2);
                st_shared_v4(dst + (((4 * half + c) ^ sw) << 4), v.x, v.y, v.z, v.w);
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[as]);
            if (++qs == qstages) {
                qs = 0;
                qph ^= 1;
            }
            if (++as == astages) {
                as = 0;
                aph ^= 1;
            }
        }
        // Y may still be in use by the previous kernel until it has finished.
        pdl_wait();

        // ---------------- epilogue
        // Warps 2-5 and 6-9 each cover the 128 channels (TMEM lane quarter
        // warp % 4) and take alternate 16-token column chunks.
        const int q = warp & 3;                    // TMEM lane quarter of this warp
        const int eh = (warp - 2) >> 2;            // which of the two warp sets
        const int ch = q * 32 + lane;
        const int n = tn * kBM + ch;
        const bool col_ok = n < p.n;
        const float bias = (col_ok && p.bias) ? p.bias[n] : 0.f;
        const bool have = my_kb > 0 && mbar_wait(&tfull_bar, 0, &abort_sh, p.status);
        if (have) tc_fence_after();
        __syncwarp();
        const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
        if (splits == 1) {
            for (int c = 16 * eh; c < NT && m0 + c < p.m; c += 32) {
                uint32_t r[16];
                tmem_ld16(tb + c, r);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int t = m0 + c + i;
                    if (have && col_ok && t < p.m) {
                        float v = __uint_as_float(r[i]);
                        if (p.bias) v = __fadd_rn(v, bias);
                        p.y[static_cast<int64_t>(t) * p.ldy + n] = __float2bfloat16_rn(v);
                    }
                }
            }
        } else if constexpr (C::SPLIT) {
            // Push this rank's partial of token t to rank t % splits, slot
            // [rank][t / splits][channel].
            const int tpo = (NT + splits - 1) / splits;
            const uint32_t red_base = smem_addr(red);
#pragma unroll
            for (int c = 16 * eh; c < NT; c += 32) {
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
        }
        __syncwarp();
    }

    if constexpr (C::SPLIT) {
        if (splits > 1) {
            __syncthreads();
            cluster_sync();
            if (warp >= 2) {
                const int q = warp & 3;
                const int eh = (warp - 2) >> 2;
                const int ch = q * 32 + lane;
                const int n = tn * kBM + ch;
                const int tpo = (NT + splits - 1) / splits;
                if (n < p.n) {
                    const float bias = p.bias ? p.bias[n] : 0.f;
                    for (int t = static_cast<int>(rank) + eh * splits; t < NT && m0 + t < p.m; t += 2 * splits) {
                        const int tl = t / splits;
                        float s = 0.f;
                        for (int r = 0; r < splits; ++r)
                            s = __fadd_rn(s, __uint_as_float(red[(r * tpo + tl) * kBM + ch]));
                        if (p.bias) s = __fadd_rn(s, bias);
                        p.y[static_cast<int64_t>(m0 + t) * p.ldy + n] = __float2bfloat16_rn(s);
                    }
                }
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

bool make_map2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
                uint64_t outer, uint64_t ld_bytes, uint32_t box_inner, uint32_t box_outer,
                CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {ld_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

template <int NT, bool BF16>
q8_status run_w4(const W4Args& a, cudaStream_t s) {
    using C = W4Cfg<NT>;
    CUtensorMap tQ, tS, tX;
    const int gps = a.group < kBK ? kBK / a.group : 1;
    if (!make_map2d(&tQ, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.codes, a.k / 2, a.n, a.ldc, kBK / 2, kBM,
                    CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map2d(&tS, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.scale, a.n, a.k / a.group, a.n * 4, kBM,
                    gps, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map2d(&tX, BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                    a.x, a.k, a.m, a.ldx * 2, kBK, NT, CU_TENSOR_MAP_SWIZZLE_128B))
        return Q8_ERR_CUDA;
    const int tiles_n = static_cast<int>((a.n + kBM - 1) / kBM);
    const int tiles_m = static_cast<int>((a.m + NT - 1) / NT);
    const int num_kb = static_cast<int>((a.k + kBK - 1) / kBK);
    int splits = 1, per = num_kb;
    int astages, qstages;
    if constexpr (C::SPLIT) {
        // Split K over a cluster (at most 8, every split non-empty) so that the
        // grid fills the SMs in one wave: two CTAs per SM for token tiles of 16
        // and 32, one for 64 (its staging and reduction buffers take more than
        // half an SM's shared memory).
        int want = (NT == 64 ? 1 : 2) * sm_count() / (tiles_n * tiles_m);
        if (want < 1) want = 1;
        if (want > 8) want = 8;
        if (want > num_kb) want = num_kb;
        per = (num_kb + want - 1) / want;
        splits = (num_kb + per - 1) / per;
        astages = NT == 64 ? 3 : 2;
        qstages = NT == 32 ? 6 : 8;
    } else {
        // Deep rings of dequantized slices: the dequantizing warps refill a
        // slot only after the MMAs that read it completed, so with two slots
        // the tensor pipe idled for that round trip on every K slice.
        astages = NT == 128 ? 5 : 4;
        qstages = NT == 128 ? 6 : 4;
    }
    if (astages > per) astages = per;
    if (qstages > per) qstages = per;
    const int smem = astages * kABytes + qstages * C::QSLOT + C::RED_BYTES + 1024;

    auto kern = w4a16_kernel<NT, BF16>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
        cudaGetLastError();
        return Q8_ERR_LAUNCH;
    }
    W4Params p;
    p.m = static_cast<int>(a.m);
    p.n = static_cast<int>(a.n);
    p.bias = a.bias;
    p.y = a.y;
    p.ldy = a.ldy;
    p.status = device_status_ptr();

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles_n), static_cast<unsigned>(splits),
                       static_cast<unsigned>(tiles_m));
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (splits > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = 1;
        attr[na].val.clusterDim.y = static_cast<unsigned>(splits);
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    if (cudaLaunchKernelEx(&cfg, kern, tQ, tS, tX, p, num_kb, per, splits, astages, qstages,
                           a.group) != cudaSuccess) {
        cudaGetLastError();
        return Q8_ERR_LAUNCH;
    }
    return Q8_OK;
}

template <bool BF16>
q8_status dispatch_w4(const W4Args& a, cudaStream_t s) {
    if (a.m <= 16) return run_w4<16, BF16>(a, s);
    if (a.m <= 32) return run_w4<32, BF16>(a, s);
    if (a.m <= 64) return run_w4<64, BF16>(a, s);
    if (a.m <= 128) return run_w4<128, BF16>(a, s);
    return run_w4<256, BF16>(a, s);
}

}  // namespace

cudaError_t launch_group_quant(const void* W, q8_dtype dt, int64_t n, int64_t k, int64_t ldw,
                               int group, uint8_t* codes, int64_t ldc, float* scale,
                               cudaStream_t s) {
    const int64_t groups = n * (k / group);
    if (groups == 0) return cudaSuccess;
    const unsigned blocks = static_cast<unsigned>((groups + 255) / 256);
    if (dt == Q8_F16)
        group_quant_kernel<__half><<<blocks, 256, 0, s>>>(static_cast<const __half*>(W), n, k, ldw,
                                                         group, codes, ldc, scale);
    else
        group_quant_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
            static_cast<const __nv_bfloat16*>(W), n, k, ldw, group, codes, ldc, scale);
    return cudaGetLastError();
}

cudaError_t launch_q4k_quant(const void* W, q8_dtype dt, int64_t n, int64_t k, int64_t ldw,
                             uint8_t* codes, int64_t ldc, float* scale, uint8_t* sub_codes,
                             float* super_scale, cudaStream_t s) {
    const int64_t blocks_total = n * (k / 256);
    if (blocks_total == 0) return cudaSuccess;
    const unsigned blocks = static_cast<unsigned>((blocks_total + 255) / 256);
    if (dt == Q8_F16)
        q4k_quant_kernel<__half><<<blocks, 256, 0, s>>>(static_cast<const __half*>(W), n, k, ldw,
                                                       codes, ldc, scale, sub_codes, super_scale);
    else
        q4k_quant_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
            static_cast<const __nv_bfloat16*>(W), n, k, ldw, codes, ldc, scale, sub_codes,
            super_scale);
    return cudaGetLastError();
}

cudaError_t launch_q4k_expand(const uint8_t* sub_codes, const float* super_scale, int64_t n,
                              int64_t k, float* scale, cudaStream_t s) {
    const int64_t total = n * (k / 32);
    if (total == 0) return cudaSuccess;
    q4k_expand_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, s>>>(sub_codes, super_scale,
                                                                                 n, k, scale);
    return cudaGetLastError();
}

q8_status launch_w4a16(const W4Args& a, cudaStream_t s) {
    if (a.m == 0 || a.n == 0) return Q8_OK;
    return a.x_bf16 ? dispatch_w4<true>(a, s) : dispatch_w4<false>(a, s);
}

}  // namespace q8
