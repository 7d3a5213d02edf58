// Tied LM head on the 5th-generation tensor cores (tcgen05, TMEM accumulators), with the
// greedy argmax fused: logits[b, n] = sum_k E[n, k] h[b, k] over the f32 token embedding E
// and the final-normed hidden rows h (cera whisper.rs / franken_ocr decoder_qwen2.rs: the
// head is tied to the embedding; argmax picks the lowest index among equal maxima).
//
// f32 products on integer tensor cores (the splitting idea of Ozaki et al., "Error-free
// transformations of matrix multiplication by using fast routines of matrix
// multiplication", 2012; and of Ootomo, Ozaki and Yokota, "DGEMM on integer matrix
// multiplication unit", 2024): every row r of E and of h is written with a per-row scale
// s_r = amax_r / 127 as three base-254 int8 digits,
//     v ~ s_r (d1 + d2 / 254 + d3 / 254^2),  |error| <= 2^-22 amax_r  (digits3 below),
// the embedding once when the weights are loaded (3 bytes per weight instead of 4), the
// hidden rows once per step (k_rowprep_digits). The six digit products whose weight is at
// least 254^-2 go through tcgen05.mma .kind::i8 with exact int32 accumulation in TMEM,
// grouped by weight into three accumulators
//     A0 = D1 E1,  A1 = D1 E2 + D2 E1,  A2 = D1 E3 + D2 E2 + D3 E1,
// and the logit is s_n s_b (A0 + (A1 + A2 / 254) / 254) in f32. The dropped products are
// below 254^-3 relative; |A| <= 3 * 127^2 * K stays inside int32 for K <= 4096. Because the
// sums are exact integers, a stream's logits do not depend on which other streams share
// the batch.
//
// CTA (192 threads, one per SM): warp 0 streams the three digit planes of 128-row
// embedding blocks with 2-D TMA loads (128 rows x 128 bytes per plane, 128-byte swizzle,
// no multicast) into a ring of 48 KB stages; warp 1 owns the TMEM allocation and issues
// the MMAs (M = 128 embedding rows, K = 32 per instruction) into one of two TMEM
// accumulator sets, committing each stage back to the producer and each block to the
// epilogue; warps 2..5 read the accumulators (tcgen05.ld, one TMEM lane quarter each),
// write the logits and keep a running argmax key per batch column. The hidden digit
// planes of the CTA's batch tile are loaded once, by TMA, in the same swizzled K-major
// layout, the three planes of each 128-column chunk stacked along N (D1 | D2 | D3, BT rows
// each) and the accumulators A0 | A1 | A2 side by side in TMEM: then E1 [D1 D2 D3]
// (N = 3 BT), E2 [D1 D2] (N = 2 BT, into A1 | A2) and E3 D1 (N = BT, into A2) are the six
// products in three instructions. An M = 128, K = 32 int8 MMA takes about 135 SM cycles
// whatever its N (measured on B200 from N = 16 to 256), so the instruction count, not the
// columns, sets the MMA time of a block.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "gemv.cuh"

namespace dec {

constexpr int kHeadThreads = 192;
constexpr int kHeadRows = 128;                      // embedding rows per block (MMA M)
constexpr int kHeadKC = 128;                        // K per stage (one 128-byte box per plane)
constexpr int kHeadPlaneBox = kHeadRows * kHeadKC;  // 16 KB
constexpr int kHeadStageBytes = 3 * kHeadPlaneBox;  // 48 KB
constexpr int kHeadMaxStages = 4;      // three-digit stages (48 KB)
constexpr int kHeadMaxStagesW1 = 8;    // one-digit stages (16 KB); sizes the stage barriers
static_assert(kHeadMaxStagesW1 >= kHeadMaxStages, "the barrier arrays hold every stage count");
constexpr int kHeadMaxK = 4096;

struct HeadArgs {
    CUtensorMap wmap;      // embedding digit planes [3 V, K] int8: box {128 bytes, 128 rows}
    CUtensorMap xmap16;    // hidden digit planes [3 MB, K] int8: box {128 bytes, 16 rows}
    CUtensorMap xmap32;    // the same with boxes of 32 rows
    const float* wscale;   // [V] embedding row scales
    const float* xscale;   // [MB] hidden row scales (hidden planes made by k_rowprep_digits)
    const float* x;        // residual rows [B, K] (hidden planes made in the head kernel)
    int x_ld;
    const float* norm_w;   // final norm
    const float* norm_b;
    float eps;
    int V, K, B, MB;
    int n_by;              // batch tiles (fastest-varying CTA index)
    float* logits;         // [B, V] or null
    unsigned long long* keys;  // [B] argmax keys, zero between launches
    int* counter;              // CTA arrival count, zero between launches
    int* argmax_out;           // [B] or null
    int* last_tok;             // [slots]
    const StepMeta* meta;
    int* err;
    // int8 head (one embedding digit): per hidden row S1 = sum |D1|, S2 = sum |D2| [MB, 2], and
    // the per-row threshold max_n (coarse_n - bound_n) written by the last CTA [B]
    const int* xsum;
    float* thr;
};

// Three base-254 digits of v / s with inv = 1 / s (|v| <= amax, so |v inv| <= 127).
__device__ __forceinline__ void digits3(float v, float inv, int& d1, int& d2, int& d3) {
    const float r0 = v * inv;
    const float e1 = fminf(fmaxf(rintf(r0), -127.0f), 127.0f);
    const float r1 = (r0 - e1) * 254.0f;
    const float e2 = fminf(fmaxf(rintf(r1), -127.0f), 127.0f);
    const float r2 = (r1 - e2) * 254.0f;
    const float e3 = fminf(fmaxf(rintf(r2), -127.0f), 127.0f);
    d1 = static_cast<int>(e1);
    d2 = static_cast<int>(e2);
    d3 = static_cast<int>(e3);
}

// One row's three digit planes, computed by one warp (the final LayerNorm / RMSNorm first
// when PRO says so, with the CUDA-core projection prologue's arithmetic): `get(j)` returns
// the row's float4 element lane + 32 j (j < jmax; elements at or past K / 4 are skipped), and
// `sink(k4, p1, p2, p3)` receives the packed digits of elements 4 k4 .. 4 k4 + 3; returns the
// row scale. Every caller uses this one function, whether the row comes from memory or from
// registers, so the digits do not depend on where they are made.
template <int PRO, class Get, class Sink>
__device__ __forceinline__ float row_digits_passes(Get get, int jmax, const float* __restrict__ gw,
                                                   const float* __restrict__ gb, float eps, int K, int lane,
                                                   Sink sink, int* s12) {
    const int K4 = K >> 2;
    float mu = 0.0f, rstd = 1.0f;
    if (PRO == PRO_LN) {
        float sum = 0.0f;
#pragma unroll
    #pragma unroll
    for (int j = 0; j < jmax; ++j)
            if (lane + 32 * j < K4) {
                const float4 v = get(j);
                sum += (v.x + v.y) + (v.z + v.w);
            }
        mu = warp_sum(sum) / static_cast<float>(K);
        float var = 0.0f;
#pragma unroll
    #pragma unroll
    for (int j = 0; j < jmax; ++j)
            if (lane + 32 * j < K4) {
                const float4 v = get(j);
                const float d0 = v.x - mu, d1 = v.y - mu, d2 = v.z - mu, d3 = v.w - mu;
                var = fmaf(d0, d0, var);
                var = fmaf(d1, d1, var);
                var = fmaf(d2, d2, var);
                var = fmaf(d3, d3, var);
            }
        var = warp_sum(var) / static_cast<float>(K);
        rstd = 1.0f / sqrtf(var + eps);
    } else if (PRO == PRO_RMS) {
        float ss = 0.0f;
#pragma unroll
    #pragma unroll
    for (int j = 0; j < jmax; ++j)
            if (lane + 32 * j < K4) {
                const float4 v = get(j);
                ss = fmaf(v.x, v.x, ss);
                ss = fmaf(v.y, v.y, ss);
                ss = fmaf(v.z, v.z, ss);
                ss = fmaf(v.w, v.w, ss);
            }
        ss = warp_sum(ss) / static_cast<float>(K);
        rstd = 1.0f / sqrtf(ss + eps);
    }
    auto normed = [&](int j) {
        float4 v = get(j);
        if (PRO != PRO_NONE) {
            const int k = lane + 32 * j;
            const float4 g = reinterpret_cast<const float4*>(gw)[k];
            float4 be = make_float4(0.f, 0.f, 0.f, 0.f);
            if (PRO == PRO_LN) be = reinterpret_cast<const float4*>(gb)[k];
            v = make_float4(norm_value(PRO, v.x, mu, rstd, g.x, be.x), norm_value(PRO, v.y, mu, rstd, g.y, be.y),
                            norm_value(PRO, v.z, mu, rstd, g.z, be.z), norm_value(PRO, v.w, mu, rstd, g.w, be.w));
        }
        return v;
    };
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < jmax; ++j)
        if (lane + 32 * j < K4) {
            const float4 v = normed(j);
            amax = fmaxf(fmaxf(amax, fabsf(v.x)), fmaxf(fabsf(v.y), fmaxf(fabsf(v.z), fabsf(v.w))));
        }
    amax = warp_max(amax);
    const float inv = amax > 0.0f ? 127.0f / amax : 0.0f;
    int sum1 = 0, sum2 = 0;
#pragma unroll
    for (int j = 0; j < jmax; ++j)
        if (lane + 32 * j < K4) {
            const float4 v = normed(j);
            const float e[4] = {v.x, v.y, v.z, v.w};
            uint32_t p1 = 0, p2 = 0, p3 = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                int d1, d2, d3;
                digits3(e[i], inv, d1, d2, d3);
                sum1 += abs(d1);
                sum2 += abs(d2);
                p1 |= (static_cast<uint32_t>(d1) & 0xffu) << (8 * i);
                p2 |= (static_cast<uint32_t>(d2) & 0xffu) << (8 * i);
                p3 |= (static_cast<uint32_t>(d3) & 0xffu) << (8 * i);
            }
            sink(lane + 32 * j, p1, p2, p3);
        }
    if (s12) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            sum1 += __shfl_xor_sync(0xffffffffu, sum1, o);
            sum2 += __shfl_xor_sync(0xffffffffu, sum2, o);
        }
        s12[0] = sum1;
        s12[1] = sum2;
    }
    return amax / 127.0f;
}

// The same for a row read from memory (x: K floats, 16-byte aligned).
template <int PRO, class Sink>
__device__ __forceinline__ float row_digits_warp(const float* __restrict__ x, const float* __restrict__ gw,
                                                 const float* __restrict__ gb, float eps, int K, int lane,
                                                 Sink sink, int* s12 = nullptr) {
    const float4* xr = reinterpret_cast<const float4*>(x);
    return row_digits_passes<PRO>([&](int j) { return xr[lane + 32 * j]; }, ((K >> 2) + 31) / 32, gw, gb, eps, K,
                                  lane, sink, s12);
}

// One logit from the three exact digit-product sums: s_n s_b (A0 + (A1 + A2 / 254) / 254), every
// f32 operation rounded on its own (no contraction), so that the head and the refine kernel of
// the int8 head give the same bits for the same sums.
__device__ __forceinline__ float digit_logit(int a0, int a1, int a2, float sn, float sb) {
    const float u = __fadd_rn(static_cast<float>(a1), __fmul_rn(static_cast<float>(a2), 1.0f / 254.0f));
    const float w = __fadd_rn(static_cast<float>(a0), __fmul_rn(u, 1.0f / 254.0f));
    return __fmul_rn(__fmul_rn(sn, sb), w);
}

// Bound on |exact - coarse| of the int8 head, where coarse uses only the embedding row's first
// digit: the dropped terms are s_n s_b (D1.E2 / 254 + (D1.E3 + D2.E2) / 254^2) with every
// embedding digit in [-127, 127], so their magnitude is at most
// s_n s_b (127 / 254 (1 + 1 / 254) S1 + 127 / 254^2 S2), S1 = sum |D1|, S2 = sum |D2| of the
// hidden row; 0.502 and 0.002 cover the two coefficients (0.50197, 0.00197), and the last term
// covers the f32 rounding of both logits (a few ulps each).
__device__ __forceinline__ float int8_head_bound(float sn, float sb, int s1, int s2, float coarse) {
    const float b = sn * sb * (0.502f * static_cast<float>(s1) + 0.002f * static_cast<float>(s2));
    return b * 1.001f + 4.0e-6f * fabsf(coarse) + 1.0e-30f;
}

// Value of an argmax key (the inverse of argmax_key's order-preserving transform).
__device__ __forceinline__ float argmax_key_value(unsigned long long k) {
    uint32_t u = static_cast<uint32_t>(k >> 32);
    u = (u & 0x80000000u) ? (u & 0x7fffffffu) : ~u;
    return __uint_as_float(u);
}

// Digit planes of rows of a row-major f32 matrix: out[p][r][k], scale[r]. One warp per
// row (the embedding and f32 projection weights once at load; the hidden rows of batches
// above 16 and the Whisper projections' input rows every step).
constexpr int kDigitsRegK4 = 12;   // rows of K <= 32 * 12 * 4 = 1536 stay in registers
template <int PRO>
__global__ void __launch_bounds__(128) k_rowprep_digits(const float* __restrict__ x, int x_ld,
                                                        const float* __restrict__ gw, const float* __restrict__ gb,
                                                        float eps, int K, int rows, long long plane_stride,
                                                        int8_t* __restrict__ out, float* __restrict__ scale,
                                                        int* __restrict__ sums) {
    // the norm's weight (and LayerNorm bias) rows do not depend on the previous kernel: they
    // are copied into shared memory before the dependency wait
    extern __shared__ float4 rd_norm[];
    const int K4 = K >> 2;
    if (PRO != PRO_NONE)
        for (int i = threadIdx.x; i < K4; i += blockDim.x) {
            rd_norm[i] = reinterpret_cast<const float4*>(gw)[i];
            if (PRO == PRO_LN) rd_norm[K4 + i] = reinterpret_cast<const float4*>(gb)[i];
        }
    pdl_launch_dependents();
    pdl_wait();
    __syncthreads();
    const float* gws = reinterpret_cast<const float*>(rd_norm);
    const float* gbs = reinterpret_cast<const float*>(rd_norm + K4);
    const int lane = threadIdx.x & 31;
    const int r = blockIdx.x * 4 + (threadIdx.x >> 5);
    if (r >= rows) return;
    uint32_t* o1 = reinterpret_cast<uint32_t*>(out + static_cast<long long>(r) * K);
    uint32_t* o2 = reinterpret_cast<uint32_t*>(out + plane_stride + static_cast<long long>(r) * K);
    uint32_t* o3 = reinterpret_cast<uint32_t*>(out + 2 * plane_stride + static_cast<long long>(r) * K);
    int s12[2];
    auto sink = [&](int k4, uint32_t p1, uint32_t p2, uint32_t p3) {
        o1[k4] = p1;
        o2[k4] = p2;
        o3[k4] = p3;
    };
    const float* xrow = x + static_cast<long long>(r) * x_ld;
    float sc;
    if (K4 <= 32 * kDigitsRegK4) {
        // the row read once into registers (every loop of the passes fully unrolled over the
        // compile-time bound); same elements, same order as the memory path
        const float4* xr = reinterpret_cast<const float4*>(xrow);
        float4 rv[kDigitsRegK4];
#pragma unroll
        for (int j = 0; j < kDigitsRegK4; ++j)
            rv[j] = lane + 32 * j < K4 ? xr[lane + 32 * j] : make_float4(0.f, 0.f, 0.f, 0.f);
        sc = row_digits_passes<PRO>([&](int j) { return rv[j]; }, kDigitsRegK4, gws, gbs, eps, K, lane, sink, s12);
    } else {
        sc = row_digits_warp<PRO>(xrow, gws, gbs, eps, K, lane, sink, s12);
    }
    if (lane == 0) {
        scale[r] = sc;
        if (sums) {
            sums[2 * r] = s12[0];
            sums[2 * r + 1] = s12[1];
        }
    }
}

// ---- tcgen05 / TMEM primitives ----------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, int8 x int8 -> int32
__device__ __forceinline__ void umma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// arrive on `bar` once every tcgen05 operation issued so far by this thread has completed
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// Shared-memory matrix descriptor of a K-major operand in the 128-byte-swizzled layout that
// TMA writes: rows of 128 bytes, 8-row groups 1024 bytes apart (stride byte offset), the
// leading byte offset unused (1), descriptor version 1, layout type 2 (SWIZZLE_128B).
__device__ __forceinline__ uint64_t smem_desc_sw128(const void* p) {
    const uint64_t addr = smem_u32(p);
    return ((addr & 0x3FFFFull) >> 4) | (1ull << 16) | (uint64_t(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor: int32 accumulator, signed int8 A and B, both K-major, N = n, M = 128.
__host__ __device__ constexpr uint32_t idesc_i8(int n) {
    return (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(kHeadRows >> 4) << 24);
}

template <int BT>
struct HeadTmemLd;
template <>
struct HeadTmemLd<8> {
    __device__ __forceinline__ static void run(uint32_t taddr, int (&r)[8]) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                     : "r"(taddr));
    }
};
template <>
struct HeadTmemLd<16> {
    __device__ __forceinline__ static void run(uint32_t taddr, int (&r)[16]) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
              "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
            : "r"(taddr));
    }
};
template <>
struct HeadTmemLd<32> {
    __device__ __forceinline__ static void run(uint32_t taddr, int (&r)[32]) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
            "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
              "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
              "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
              "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
            : "r"(taddr));
    }
};
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// XPRO: kHeadXExternal when k_rowprep_digits made the hidden planes (read by TMA), else the
// final norm (PRO_LN / PRO_RMS) with which this kernel makes them itself.
constexpr int kHeadXExternal = -1;

// WD: embedding digits streamed and multiplied, 3 (the exact head) or 1 (the int8 head: coarse
// logits from the first digit, the per-row int8 quantisation of the embedding, plus the bound
// that selects the candidates k_head_refine recomputes exactly).
template <int BT, int XPRO, int WD>
__global__ void __launch_bounds__(kHeadThreads, 1) k_head_tc(const __grid_constant__ HeadArgs A, int NS) {
    static_assert(BT == 16 || BT == 32, "batch tile");
    static_assert(WD == 1 || WD == 3, "embedding digits");
    static_assert(WD == 3 || XPRO == kHeadXExternal, "the int8 head reads the hidden planes k_rowprep_digits made");
    constexpr int kStage = WD * kHeadPlaneBox;
    constexpr int ACC = 3 * BT;                           // TMEM columns of one accumulator set
    constexpr uint32_t TCOLS = BT == 16 ? 128 : 256;      // two sets, power of two
    constexpr int XC = 3 * BT * 128;                      // one chunk of the three stacked hidden planes
    constexpr uint32_t IDESC1 = idesc_i8(3 * BT);         // E1 against D1 | D2 | D3
    constexpr uint32_t IDESC2 = idesc_i8(2 * BT);         // E2 against D1 | D2
    constexpr uint32_t IDESC3 = idesc_i8(BT);             // E3 against D1
    const int nch = (A.K + kHeadKC - 1) / kHeadKC;
    const int xplane = nch * BT * 128;                    // bytes of one hidden digit plane (all chunks)

    extern __shared__ unsigned char head_smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(head_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    unsigned char* ring = smem;                                             // NS stages
    unsigned char* sx = smem + static_cast<size_t>(NS) * kStage;            // nch chunks of XC bytes
    __shared__ __align__(8) uint64_t full[kHeadMaxStagesW1], empty[kHeadMaxStagesW1];   // NS <= 8 stages
    __shared__ __align__(8) uint64_t tfull[2], tempty[2], bar_x, bar_done;
    __shared__ uint32_t s_tmem;
    __shared__ unsigned long long s_key[BT];
    __shared__ float s_xs[BT];
    __shared__ int s_sum1[BT], s_sum2[BT];
    __shared__ int s_fail, s_last;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_by = A.n_by;
    const int by = blockIdx.x % n_by, b0 = by * BT;
    const int nb = min(BT, A.B - b0);
    const int n_blocks = (A.V + kHeadRows - 1) / kHeadRows;
    const int cps = gridDim.x / n_by;
    const int c0 = blockIdx.x / n_by;
    const int my_blocks = c0 < n_blocks ? (n_blocks - 1 - c0) / cps + 1 : 0;
    const int n_items = my_blocks * nch;

    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 4);
        }
        mbar_init(&bar_x, 1);
        mbar_init(&bar_done, 1);
        mbar_fence_init();
        s_fail = 0;
    }
    if (tid < BT) s_key[tid] = 0ull;
    if (warp == 1) {
        tmem_alloc(&s_tmem, TCOLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = s_tmem;

    // weights do not depend on earlier kernels: the first stages go out before the wait
    auto issue = [&](int it) {
        const int jb = c0 + (it / nch) * cps;
        const int c = it % nch;
        unsigned char* dst = ring + static_cast<size_t>(it % NS) * kStage;
        mbar_arrive_expect_tx(&full[it % NS], kStage);
#pragma unroll
        for (int p = 0; p < WD; ++p)
            tma_load_2d(dst + p * kHeadPlaneBox, &A.wmap, c * kHeadKC, p * A.V + jb * kHeadRows, &full[it % NS]);
    };
    int n_issued = 0;
    if (warp == 0 && lane == 0)
        for (; n_issued < NS && n_issued < n_items; ++n_issued) issue(n_issued);
    pdl_launch_dependents();
    pdl_wait();

    if (XPRO == kHeadXExternal) {
        if (tid < BT) {
            s_xs[tid] = tid < nb ? A.xscale[b0 + tid] : 0.0f;
            if (WD == 1) {
                s_sum1[tid] = tid < nb ? A.xsum[2 * (b0 + tid)] : 0;
                s_sum2[tid] = tid < nb ? A.xsum[2 * (b0 + tid) + 1] : 0;
            }
        }
    } else {
        // the hidden planes in the swizzled K-major layout the MMA reads: zero first (rows past
        // the batch, columns past K), then one warp per row writes its digits
        for (int o = tid * 16; o < 3 * xplane; o += kHeadThreads * 16)
            *reinterpret_cast<uint4*>(sx + o) = make_uint4(0u, 0u, 0u, 0u);
        if (tid < BT) s_xs[tid] = 0.0f;
        __syncthreads();
        for (int b = warp; b < nb; b += kHeadThreads / 32) {
            const float sc = row_digits_warp<(XPRO < 0 ? PRO_NONE : XPRO)>(
                A.x + static_cast<long long>(b0 + b) * A.x_ld, A.norm_w, A.norm_b, A.eps, A.K, lane,
                [&](int k4, uint32_t p1, uint32_t p2, uint32_t p3) {
                    const int j = (4 * k4) & 127;   // byte within the 128-byte row of chunk (4 k4) / 128
                    const int off = ((4 * k4) >> 7) * XC + b * 128 + (((j >> 4) ^ (b & 7)) << 4) + (j & 15);
                    *reinterpret_cast<uint32_t*>(sx + off) = p1;
                    *reinterpret_cast<uint32_t*>(sx + BT * 128 + off) = p2;
                    *reinterpret_cast<uint32_t*>(sx + 2 * BT * 128 + off) = p3;
                });
            if (lane == 0) s_xs[b] = sc;
        }
        // generic-proxy shared-memory writes become visible to the tensor core
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();
    if (warp == 0 && lane == 0) {
        if (XPRO == kHeadXExternal) {
            // hidden digit planes of this batch tile (written by k_rowprep_digits)
            mbar_arrive_expect_tx(&bar_x, 3 * xplane);
            for (int p = 0; p < 3; ++p)
                for (int c = 0; c < nch; ++c)
                    tma_load_2d(sx + c * XC + p * BT * 128, BT == 16 ? &A.xmap16 : &A.xmap32, c * kHeadKC,
                                p * A.MB + b0, &bar_x);
        }
        // remaining weight stages
        for (int it = n_issued; it < n_items; ++it) {
            if (!mbar_wait_bounded(&empty[it % NS], static_cast<uint32_t>(it / NS - 1) & 1u, A.err)) {
                s_fail = 1;
                break;
            }
            issue(it);
            n_issued = it + 1;
        }
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issuer ----
        bool ok = XPRO != kHeadXExternal || mbar_wait_bounded(&bar_x, 0, A.err);
        tc_fence_after();
        int it = 0;
        for (int i = 0; ok && i < my_blocks; ++i) {
            const int ab = i & 1;
            if (i >= 2 && !mbar_wait_bounded(&tempty[ab], static_cast<uint32_t>((i >> 1) - 1) & 1u, A.err)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t dacc = tbase + static_cast<uint32_t>(ab * (TCOLS / 2));
            for (int c = 0; c < nch; ++c, ++it) {
                const int stage = it % NS;
                if (!mbar_wait_bounded(&full[stage], static_cast<uint32_t>(it / NS) & 1u, A.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const unsigned char* st = ring + static_cast<size_t>(stage) * kStage;
#pragma unroll
                for (int s = 0; s < kHeadKC / 32; ++s) {
                    const uint64_t w1 = smem_desc_sw128(st) + 2 * s;
                    // the chunk's hidden planes D1 | D2 | D3 stacked along N; the accumulators
                    // A0 | A1 | A2 side by side in TMEM
                    const uint64_t xs = smem_desc_sw128(sx + c * XC) + 2 * s;
                    const uint32_t first = (c == 0 && s == 0) ? 0u : 1u;
                    // E1 D1 -> A0, E1 D2 -> A1, E1 D3 -> A2 (the int8 head stops here)
                    umma_i8(dacc, w1, xs, IDESC1, first);
                    if (WD == 3) {
                        // E2 D1 -> A1, E2 D2 -> A2; E3 D1 -> A2
                        const uint64_t w2 = smem_desc_sw128(st + kHeadPlaneBox) + 2 * s,
                                       w3 = smem_desc_sw128(st + 2 * kHeadPlaneBox) + 2 * s;
                        umma_i8(dacc + BT, w2, xs, IDESC2, 1u);
                        umma_i8(dacc + 2 * BT, w3, xs, IDESC3, 1u);
                    }
                }
                umma_commit(&empty[stage]);   // stage free once these MMAs have read it
            }
            if (!ok) break;
            umma_commit(&tfull[ab]);          // accumulator set ready for the epilogue
        }
        if (!ok) s_fail = 1;
        // every MMA issued has completed before TMEM is released
        umma_commit(&bar_done);
        mbar_wait_bounded(&bar_done, 0, nullptr);
    } else if (warp >= 2) {
        // ---- epilogue: TMEM lane quarter q holds embedding rows 32 q .. 32 q + 31 ----
        const int q = warp & 3;
        unsigned long long best[BT];
#pragma unroll
        for (int b = 0; b < BT; ++b) best[b] = 0ull;
        for (int i = 0; i < my_blocks; ++i) {
            const int ab = i & 1;
            if (!mbar_wait_bounded(&tfull[ab], static_cast<uint32_t>(i >> 1) & 1u, A.err)) {
                s_fail = 1;
                break;
            }
            tc_fence_after();
            const uint32_t t0 = tbase + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(ab * (TCOLS / 2));
            int a0[BT], a1[BT], a2[BT];
            HeadTmemLd<BT>::run(t0, a0);
            HeadTmemLd<BT>::run(t0 + BT, a1);
            HeadTmemLd<BT>::run(t0 + 2 * BT, a2);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[ab]);
            const int jb = c0 + i * cps;
            const int n = jb * kHeadRows + q * 32 + lane;
            if (n < A.V) {
                const float sn = __ldg(A.wscale + n);
#pragma unroll
                for (int b = 0; b < BT; ++b) {
                    if (b >= nb) break;
                    const float y = digit_logit(a0[b], a1[b], a2[b], sn, s_xs[b]);
                    if (A.logits) A.logits[static_cast<long long>(b0 + b) * A.V + n] = y;
                    // the exact head ranks the logits; the int8 head ranks each logit's lower
                    // bound, whose maximum is the candidates' threshold
                    const float r = WD == 3 ? y : y - int8_head_bound(sn, s_xs[b], s_sum1[b], s_sum2[b], y);
                    const unsigned long long key = argmax_key(r, n);
                    best[b] = key > best[b] ? key : best[b];
                }
            }
        }
#pragma unroll
        for (int b = 0; b < BT; ++b) {
            unsigned long long v = best[b];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, off);
                v = o > v ? o : v;
            }
            if (lane == 0 && b < nb && v != 0ull) atomicMax(&s_key[b], v);
        }
    }
    // in-flight weight copies land before the CTA can exit
    if (warp == 0 && lane == 0 && s_fail)
        for (int i2 = max(0, n_issued - NS); i2 < n_issued; ++i2)
            mbar_wait_bounded(&full[i2 % NS], static_cast<uint32_t>(i2 / NS) & 1u, nullptr);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, TCOLS);
    }
    // fold into the grid-wide keys; the last CTA writes the picks and resets the keys
    if (tid < nb && s_key[tid] != 0ull) atomicMax(&A.keys[b0 + tid], s_key[tid]);
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        s_last = (atomicAdd(A.counter, 1) == static_cast<int>(gridDim.x) - 1);
    }
    __syncthreads();
    if (s_last) {
        __threadfence();
        for (int b = tid; b < A.B; b += kHeadThreads) {
            const unsigned long long k = atomicExch(&A.keys[b], 0ull);
            if (WD == 1) {
                A.thr[b] = (k == 0ull) ? -INFINITY : argmax_key_value(k);
                continue;
            }
            const int idx = (k == 0ull) ? 0 : argmax_key_index(k);
            if (A.argmax_out) A.argmax_out[b] = idx;
            if (A.last_tok) A.last_tok[A.meta->slot[b]] = idx;
        }
        if (tid == 0) *A.counter = 0;
    }
}

// ---------------------------------------------------------------- host side

inline size_t head_tc_smem(int K, int bt, int ns, int wd = 3) {
    const int nch = (K + kHeadKC - 1) / kHeadKC;
    return 1024 + size_t(ns) * wd * kHeadPlaneBox + size_t(3) * nch * bt * 128;
}
// stages that fit next to the hidden planes (0: the head does not fit)
inline int head_tc_stages(int K, int bt, int wd = 3) {
    if (K % 16 != 0 || K > kHeadMaxK) return 0;
    for (int ns = wd == 1 ? kHeadMaxStagesW1 : kHeadMaxStages; ns >= 2; --ns)
        if (head_tc_smem(K, bt, ns, wd) <= size_t(227 * 1024 - 1024)) return ns;   // room for static smem
    return 0;
}

template <int PRO>
cudaError_t rowprep_digits_launch(const float* x, int x_ld, const float* gw, const float* gb, float eps, int K,
                                  int rows, long long plane_stride, int8_t* out, float* scale, int* sums, bool pdl,
                                  cudaStream_t st);
// pro: the final norm when the head kernel makes the hidden planes itself (batches up to
// 16), kHeadXExternal when k_rowprep_digits made them
cudaError_t head_tc_launch(int num_sms, const HeadArgs& a, int pro, cudaStream_t st);
// The int8 head: coarse logits and thresholds (k_head_tc with one embedding digit, hidden
// planes from k_rowprep_digits), candidate selection, exact refine and the greedy pick.
// cand holds B * V ints; ncand and counter are zero between launches.
cudaError_t head_int8_launch(int num_sms, const HeadArgs& a, const int8_t* wdig, const int8_t* xdig, int* cand,
                             int* ncand, int* refine_counter, cudaStream_t st);
inline bool head_tc_makes_planes(int B) { return B <= 16; }

#ifdef DEC_HEAD_TC_DEFINE

// ---- int8 head: candidates and their exact logits ----------------------------------

// Candidates of the int8 head: every n whose coarse logit plus its bound reaches the row's
// threshold (the largest lower bound). The exact logit of every n is within the bound of its
// coarse one, so every n that can hold the exact maximum (ties included) is a candidate.
// Appended as b * V + n to `cand` (capacity B * V), counted in *ncand.
__global__ void __launch_bounds__(256) k_head_select(const float* __restrict__ logits, const float* __restrict__ wscale,
                                                     const float* __restrict__ xscale, const int* __restrict__ xsum,
                                                     const float* __restrict__ thr, int V, int* __restrict__ cand,
                                                     int* __restrict__ ncand) {
    pdl_launch_dependents();
    pdl_wait();
    const int b = blockIdx.y;
    const float sb = xscale[b], t = thr[b];
    const int s1 = xsum[2 * b], s2 = xsum[2 * b + 1];
    const int lane = threadIdx.x & 31;
    for (int n0 = blockIdx.x * blockDim.x; n0 < V; n0 += gridDim.x * blockDim.x) {
        const int n = n0 + threadIdx.x;
        bool hit = false;
        if (n < V) {
            const float y = logits[static_cast<long long>(b) * V + n];
            hit = y + int8_head_bound(__ldg(wscale + n), sb, s1, s2, y) >= t;
        }
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        if (m == 0u) continue;
        int base = 0;
        if (lane == 0) base = atomicAdd(ncand, __popc(m));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (hit) cand[base + __popc(m & ((1u << lane) - 1u))] = b * V + n;
    }
}

// Exact logits of the candidates (one warp each, the exact head's digit products summed with
// dp4a and combined by digit_logit: the same bits as the three-digit head), written over the
// coarse ones, then the greedy pick among them; the last CTA writes the picks and resets.
__global__ void __launch_bounds__(256) k_head_refine(const int8_t* __restrict__ wdig, const float* __restrict__ wscale,
                                                     const int8_t* __restrict__ xdig, const float* __restrict__ xscale,
                                                     long long wplane, long long xplane, int V, int K, int B,
                                                     const int* __restrict__ cand, int* __restrict__ ncand,
                                                     float* __restrict__ logits, unsigned long long* __restrict__ keys,
                                                     int* __restrict__ counter, int* __restrict__ argmax_out,
                                                     int* __restrict__ last_tok, const StepMeta* __restrict__ meta) {
    pdl_launch_dependents();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nw = (gridDim.x * blockDim.x) >> 5;
    const int total = *ncand;
    for (int c = gw; c < total; c += nw) {
        const int code = cand[c];
        const int b = code / V, n = code - b * V;
        const int8_t* e1 = wdig + static_cast<long long>(n) * K;
        const int8_t* h1 = xdig + static_cast<long long>(b) * K;
        int a0 = 0, a1 = 0, a2 = 0;
        for (int k = lane * 16; k < K; k += 32 * 16) {
            const int4 E1 = *reinterpret_cast<const int4*>(e1 + k);
            const int4 E2 = *reinterpret_cast<const int4*>(e1 + wplane + k);
            const int4 E3 = *reinterpret_cast<const int4*>(e1 + 2 * wplane + k);
            const int4 D1 = *reinterpret_cast<const int4*>(h1 + k);
            const int4 D2 = *reinterpret_cast<const int4*>(h1 + xplane + k);
            const int4 D3 = *reinterpret_cast<const int4*>(h1 + 2 * xplane + k);
            const int e1v[4] = {E1.x, E1.y, E1.z, E1.w}, e2v[4] = {E2.x, E2.y, E2.z, E2.w},
                      e3v[4] = {E3.x, E3.y, E3.z, E3.w};
            const int d1v[4] = {D1.x, D1.y, D1.z, D1.w}, d2v[4] = {D2.x, D2.y, D2.z, D2.w},
                      d3v[4] = {D3.x, D3.y, D3.z, D3.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                a0 = __dp4a(e1v[j], d1v[j], a0);
                a1 = __dp4a(e1v[j], d2v[j], a1);
                a1 = __dp4a(e2v[j], d1v[j], a1);
                a2 = __dp4a(e1v[j], d3v[j], a2);
                a2 = __dp4a(e2v[j], d2v[j], a2);
                a2 = __dp4a(e3v[j], d1v[j], a2);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            a0 += __shfl_xor_sync(0xffffffffu, a0, o);
            a1 += __shfl_xor_sync(0xffffffffu, a1, o);
            a2 += __shfl_xor_sync(0xffffffffu, a2, o);
        }
        if (lane == 0) {
            const float y = digit_logit(a0, a1, a2, __ldg(wscale + n), xscale[b]);
            logits[static_cast<long long>(b) * V + n] = y;
            atomicMax(&keys[b], argmax_key(y, n));
        }
    }
    __shared__ int s_last;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        s_last = (atomicAdd(counter, 1) == static_cast<int>(gridDim.x) - 1);
    }
    __syncthreads();
    if (s_last) {
        __threadfence();
        for (int b = threadIdx.x; b < B; b += blockDim.x) {
            const unsigned long long k = atomicExch(&keys[b], 0ull);
            const int idx = (k == 0ull) ? 0 : argmax_key_index(k);
            if (argmax_out) argmax_out[b] = idx;
            if (last_tok) last_tok[meta->slot[b]] = idx;
        }
        if (threadIdx.x == 0) {
            *counter = 0;
            *ncand = 0;
        }
    }
}


template <int PRO>
cudaError_t rowprep_digits_launch(const float* x, int x_ld, const float* gw, const float* gb, float eps, int K,
                                  int rows, long long plane_stride, int8_t* out, float* scale, int* sums, bool pdl,
                                  cudaStream_t st) {
    if (K % 4 != 0 || rows <= 0) return cudaErrorInvalidValue;
    const size_t smem = size_t(K) * 4 * (PRO == PRO_LN ? 2 : (PRO == PRO_RMS ? 1 : 0));
    if (smem > size_t(227 * 1024)) return cudaErrorInvalidValue;
    thread_local int attr_dev = -1;
    const cudaError_t e = prefer_max_shared_once(k_rowprep_digits<PRO>, attr_dev, 227 * 1024);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((rows + 3) / 4);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k_rowprep_digits<PRO>, x, x_ld, gw, gb, eps, K, rows, plane_stride, out, scale,
                              sums);
}

template <int BT, int XPRO, int WD = 3>
cudaError_t head_tc_launch_bt(int num_sms, HeadArgs a, cudaStream_t st) {
    const int ns = head_tc_stages(a.K, BT, WD);
    if (ns == 0) return cudaErrorNotSupported;
    const size_t smem = head_tc_smem(a.K, BT, ns, WD);
    thread_local int attr_dev = -1;   // attributes are per device; set again when it changes
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (attr_dev != dev) {
        e = cudaFuncSetAttribute(k_head_tc<BT, XPRO, WD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 227 * 1024 - 1024);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(k_head_tc<BT, XPRO, WD>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        attr_dev = dev;
    }
    const int gy = (a.B + BT - 1) / BT;
    a.n_by = gy;
    const int n_blocks = (a.V + kHeadRows - 1) / kHeadRows;
    const int cps = std::max(1, std::min(n_blocks, num_sms / gy));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cps * gy);
    cfg.blockDim = dim3(kHeadThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_head_tc<BT, XPRO, WD>, a, ns);
}

cudaError_t head_tc_launch(int num_sms, const HeadArgs& a, int pro, cudaStream_t st) {
    if (a.B < 1 || a.B > a.MB) return cudaErrorInvalidValue;
    if (head_tc_makes_planes(a.B)) {
        if (pro == PRO_LN) return head_tc_launch_bt<16, PRO_LN>(num_sms, a, st);
        if (pro == PRO_RMS) return head_tc_launch_bt<16, PRO_RMS>(num_sms, a, st);
        return cudaErrorInvalidValue;
    }
    if (pro != kHeadXExternal) return cudaErrorInvalidValue;
    return head_tc_launch_bt<32, kHeadXExternal>(num_sms, a, st);
}

template <typename K, typename... Args>
cudaError_t head_pdl_launch(K kern, dim3 grid, dim3 block, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

cudaError_t head_int8_launch(int num_sms, const HeadArgs& a, const int8_t* wdig, const int8_t* xdig, int* cand,
                             int* ncand, int* refine_counter, cudaStream_t st) {
    if (a.B < 1 || a.B > a.MB || a.logits == nullptr || a.thr == nullptr || a.xsum == nullptr || a.K % 16 != 0)
        return cudaErrorInvalidValue;
    cudaError_t e = a.B <= 16 ? head_tc_launch_bt<16, kHeadXExternal, 1>(num_sms, a, st)
                              : head_tc_launch_bt<32, kHeadXExternal, 1>(num_sms, a, st);
    if (e != cudaSuccess) return e;
    const int chunks = std::max(1, std::min((a.V + 255) / 256, (2 * num_sms + a.B - 1) / a.B));
    e = head_pdl_launch(k_head_select, dim3(chunks, a.B), dim3(256), st, static_cast<const float*>(a.logits),
                        a.wscale, a.xscale, a.xsum, static_cast<const float*>(a.thr), a.V, cand, ncand);
    if (e != cudaSuccess) return e;
    return head_pdl_launch(k_head_refine, dim3(num_sms), dim3(256), st, wdig, a.wscale, xdig, a.xscale,
                           static_cast<long long>(a.V) * a.K, static_cast<long long>(a.MB) * a.K, a.V, a.K, a.B,
                           static_cast<const int*>(cand), ncand, a.logits, a.keys, refine_counter, a.argmax_out,
                           a.last_tok, a.meta);
}

#endif  // DEC_HEAD_TC_DEFINE

}  // namespace dec
