// Tensor-core projections for batches of 8 to 64 streams with f32 activations: f32
// weights or int8 per-row weights (W8A32). y[b, n] = sum_k x[b, k] W[n, k].
//
// At these batch sizes the CUDA-core path needs 8-64 FMAs per weight element and runs
// out of issue slots before HBM does, so the dot products go to the tensor cores
// (mma.sync m16n8k8, TF32 operands, f32 accumulation). To keep f32 accuracy the
// activations are split as x = x_hi + x_lo (TF32 each) as they are read from shared
// memory, and f32 weights the same way; the product is x_hi w_hi + x_lo w_hi + x_hi w_lo (the
// lo*lo term is below f32 rounding). A norm prologue needs whole-row statistics, which
// one K slice does not see, so normalised rows come from k_rowprep, one CTA per row. int8 weights are exact in TF32, so they need the
// two x terms only, and the per-row scale is applied after accumulation
// (lattice-inference cpu_q8.rs, matmul_bt_q8: y_n = s_n * sum_k q_nk x_k).
//
// Decomposition: 128-row weight blocks x K slices. The CTAs form n_ks groups; group ks
// owns K slice ks and walks the row blocks, so each CTA stages its activation slice
// once. Within a CTA, 4 consumer warps own 32 rows each (two m16 tiles) x all batch
// columns (BT/8 n8 tiles): every partial output lands in one thread. One producer warp
// moves weights with 2-D TMA loads (boxes of 128 rows x 128 bytes, 128-byte swizzle, no
// multicast) into a ring of 32 KB stages with full/empty mbarriers; the first stages are
// issued before the programmatic-dependent-launch wait. With more than one slice, each
// CTA writes its partial tile to scratch, and for each warp's 32 rows the last of the
// n_ks warps that own them (an arrival count; nothing waits) sums the slices in slice
// order -- deterministic -- and runs the epilogue.
// Operand pairing: inside a 32-element K group, MMA steps 2h and 2h + 1 of quad thread t
// take four adjacent physical columns (mma_pcol); step 2h + j pairs logical k = t and
// t + 4 with the columns 2j and 2j + 1 of that group, for both operands, so every operand
// read is one shared load free of bank conflicts under the swizzle (weights) or the
// padding (activations).
#pragma once

#include <cuda.h>

#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "gemv.cuh"

namespace dec {

constexpr int kMmaConsumerWarps = 4;
constexpr int kMmaThreads = (kMmaConsumerWarps + 1) * 32;
constexpr int kMmaBlockRows = 32 * kMmaConsumerWarps;           // 128
constexpr int kMmaBoxBytes = kMmaBlockRows * 128;               // 16 KB: 128 rows x 128 bytes
constexpr int kMmaBoxesPerStage = 2;                              // int8 tensor-core kernel
constexpr int kMmaStageBytes = kMmaBoxBytes * kMmaBoxesPerStage;  // 32 KB
constexpr int kMmaMaxStages = 6;
constexpr int kMmaMaxStagesTF = 12;   // TF32 kernel: stages of one or two boxes

struct MmaArgs {
    CUtensorMap tmap;        // weights [N, K]: box {128 bytes of K, 128 rows}, 128-byte swizzle
    void* part;              // split-K partial tiles
    int* cnt;                // split-K arrival counts per (row block, batch tile, warp), zero between launches
    int n_ks;                // K slices (CTA groups)
    int ksl;                 // K elements per slice, a multiple of the stage's K
    int n_by;                // batch tiles (the fastest-varying CTA index)
    GemvArgs g;              // shapes, f32 activations (g.x, g.x_ld) and epilogue arguments
};

__device__ __forceinline__ uint32_t tf32_of(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four weight values at physical columns (byte_off / elt).. of local row `lr` of a
// 128-byte-swizzled box (16-byte chunk c of row r sits at chunk c ^ (r mod 8)).
template <typename WT>
__device__ __forceinline__ float4 load_w4(const unsigned char* box, int lr, int byte_off) {
    const int chunk = byte_off >> 4, inner = byte_off & 15;
    const unsigned char* p = box + lr * 128 + ((chunk ^ (lr & 7)) << 4) + inner;
    if (std::is_same<WT, float>::value) {
        return *reinterpret_cast<const float4*>(p);
    } else {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
        return make_float4(static_cast<float>(static_cast<int>(w << 24) >> 24),
                           static_cast<float>(static_cast<int>(w << 16) >> 24),
                           static_cast<float>(static_cast<int>(w << 8) >> 24),
                           static_cast<float>(static_cast<int>(w) >> 24));
    }
}

// Physical column group (4 columns) of quad thread t for MMA steps 2h, 2h + 1 within a
// 32-column K group, and the activation row padding that keeps the matching 16-byte
// shared loads conflict-free: f32 weights read 16 bytes at 32t + 16h of a 128-byte
// swizzled row, int8 weights 4 bytes at 16h + 4t.
template <typename WT>
__host__ __device__ constexpr int mma_pcol(int t, int h) {
    return std::is_same<WT, float>::value ? 8 * t + 4 * h : 16 * h + 4 * t;
}
template <typename WT>
__host__ __device__ constexpr int mma_xpad() {
    return std::is_same<WT, float>::value ? 4 : 16;
}

// One normalised activation row (LayerNorm or RMSNorm, the same arithmetic as the
// CUDA-core projection prologue). One CTA per row; the row is staged in shared memory
// (K <= kRowprepMaxK).
constexpr int kRowprepMaxK = 8192;
constexpr int kRowprepThreads = 256;

template <int PRO>
__global__ void __launch_bounds__(kRowprepThreads) k_rowprep(const float* __restrict__ x, int x_ld,
                                                             const float* __restrict__ g,
                                                             const float* __restrict__ beta, float eps, int K,
                                                             float* __restrict__ out) {
    __shared__ __align__(16) float row[kRowprepMaxK];
    __shared__ float red[kRowprepThreads / 32];
    __shared__ float s_stat[2];
    constexpr int NW = kRowprepThreads / 32;
    pdl_launch_dependents();
    pdl_wait();
    const int b = blockIdx.x, tid = threadIdx.x;
    const float4* xr = reinterpret_cast<const float4*>(x + static_cast<long long>(b) * x_ld);
    const int K4 = K >> 2;
    float acc = 0.0f;
    for (int k = tid; k < K4; k += kRowprepThreads) {
        const float4 v = xr[k];
        reinterpret_cast<float4*>(row)[k] = v;
        if (PRO == PRO_LN) acc += (v.x + v.y) + (v.z + v.w);
        if (PRO == PRO_RMS) acc = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, acc))));
    }
    acc = warp_sum(acc);
    if ((tid & 31) == 0) red[tid >> 5] = acc;
    __syncthreads();
    if (tid == 0) {
        float s = 0.0f;
        for (int i = 0; i < NW; ++i) s += red[i];
        s_stat[0] = s / static_cast<float>(K);
    }
    __syncthreads();
    float mu = 0.0f, rstd;
    if (PRO == PRO_LN) {
        mu = s_stat[0];
        float var = 0.0f;
        for (int k = tid; k < K4; k += kRowprepThreads) {
            const float4 v = reinterpret_cast<const float4*>(row)[k];
            const float d0 = v.x - mu, d1 = v.y - mu, d2 = v.z - mu, d3 = v.w - mu;
            var = fmaf(d0, d0, fmaf(d1, d1, fmaf(d2, d2, fmaf(d3, d3, var))));
        }
        var = warp_sum(var);
        if ((tid & 31) == 0) red[tid >> 5] = var;
        __syncthreads();
        if (tid == 0) {
            float s = 0.0f;
            for (int i = 0; i < NW; ++i) s += red[i];
            s_stat[1] = 1.0f / sqrtf(s / static_cast<float>(K) + eps);
        }
    } else {
        if (tid == 0) s_stat[1] = 1.0f / sqrtf(s_stat[0] + eps);
    }
    __syncthreads();
    rstd = s_stat[1];
    float4* o = reinterpret_cast<float4*>(out + static_cast<long long>(b) * K);
    for (int k = tid; k < K4; k += kRowprepThreads) {
        float4 v = reinterpret_cast<const float4*>(row)[k];
        const float4 gg = __ldg(reinterpret_cast<const float4*>(g) + k);
        float4 bb = make_float4(0.f, 0.f, 0.f, 0.f);
        if (PRO == PRO_LN) bb = __ldg(reinterpret_cast<const float4*>(beta) + k);
        v.x = norm_value(PRO, v.x, mu, rstd, gg.x, bb.x);
        v.y = norm_value(PRO, v.y, mu, rstd, gg.y, bb.y);
        v.z = norm_value(PRO, v.z, mu, rstd, gg.z, bb.z);
        v.w = norm_value(PRO, v.w, mu, rstd, gg.w, bb.w);
        o[k] = v;
    }
}

// NBX: 128-byte boxes per stage (1 for int8 weights, 2 for f32)
template <int BT, typename WT, int EPI, int NBX>
__global__ void __launch_bounds__(kMmaThreads, 1) k_proj_mma(const __grid_constant__ MmaArgs A, int NS) {
    const GemvArgs& a = A.g;
    constexpr int NT = BT / 8;
    constexpr int ELT = sizeof(WT);
    constexpr int BOXK = 128 / ELT;                       // K elements per box row
    constexpr int KC = BOXK * NBX;                        // K elements per stage
    constexpr int SB = kMmaBoxBytes * NBX;                // stage bytes
    constexpr bool F32W = std::is_same<WT, float>::value;
    static_assert(BT % 8 == 0, "batch tile must be a multiple of 8");

    extern __shared__ unsigned char mma_smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(mma_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    unsigned char* ring = smem;
    const int XS = A.ksl + mma_xpad<WT>();   // padded activation row (floats)
    float* sX = reinterpret_cast<float*>(smem + static_cast<size_t>(NS) * SB);
    __shared__ __align__(8) uint64_t full[kMmaMaxStagesTF];
    __shared__ __align__(8) uint64_t empty[kMmaMaxStagesTF];
    __shared__ __align__(8) uint64_t bar_x;
    __shared__ unsigned long long s_key[BT];
    __shared__ int s_slot[BT], s_len[BT];   // EPI_QKV: cache page and row in it of each column's new row
    __shared__ int s_flag, s_last;   // staging succeeded; this CTA arrived last (head)

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool producer = warp == kMmaConsumerWarps;
    // batch tile fastest, so that the tiles of one weight block read it together
    const int n_by = A.n_by;
    const int by = blockIdx.x % n_by, b0 = by * BT;
    const int nb = min(BT, a.B - b0);
    const int n_blocks = (a.N + kMmaBlockRows - 1) / kMmaBlockRows;
    const int rest = blockIdx.x / n_by;
    const int ks = rest % A.n_ks;
    const int cps = gridDim.x / (A.n_ks * n_by);         // CTAs per (K slice, batch tile)
    const int c0 = rest / A.n_ks;
    const int kstart = ks * A.ksl;
    const int klen = min(A.ksl, a.K - kstart);
    const int nkc = (klen + KC - 1) / KC;
    const int my_blocks = (c0 < n_blocks && cps > 0) ? (n_blocks - 1 - c0) / cps + 1 : 0;
    const int n_items = my_blocks * nkc;

    auto issue = [&](int it) {
        const int jb = c0 + (it / nkc) * cps;
        const int c = it % nkc;
        const int stage = it % NS;
        unsigned char* dst = ring + static_cast<size_t>(stage) * SB;
        mbar_arrive_expect_tx(&full[stage], SB);
#pragma unroll
        for (int bx = 0; bx < NBX; ++bx)
            tma_load_2d(dst + bx * kMmaBoxBytes, &A.tmap, kstart + c * KC + bx * BOXK, jb * kMmaBlockRows,
                        &full[stage]);
    };

    int n_issued = 0;
    if (producer && lane == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kMmaConsumerWarps);
        }
        mbar_init(&bar_x, 1);
        mbar_fence_init();
        for (; n_issued < NS && n_issued < n_items; ++n_issued) issue(n_issued);
    }
    pdl_launch_dependents();
    pdl_wait();

    // ---- activation slice: one bulk copy per row, then the TF32 split in place ----
    if (producer && lane == 0) {
        const uint32_t row_bytes = static_cast<uint32_t>(klen) * 4;
        mbar_arrive_expect_tx(&bar_x, row_bytes * nb);
        for (int b = 0; b < nb; ++b)
            bulk_g2s(sX + static_cast<size_t>(b) * XS, a.x + static_cast<long long>(b0 + b) * a.x_ld + kstart,
                     row_bytes, &bar_x);
        s_flag = mbar_wait_bounded(&bar_x, 0, a.err) ? 1 : 0;
    }
    if (EPI == EPI_HEAD && tid < BT) s_key[tid] = 0ull;
    if (EPI == EPI_QKV && tid < BT) {
        // the cache page and row within it of this step's new row, per batch column
        int page = 0, r = 0;
        if (tid < nb) kv_page_of(a.kv, a.meta->slot[b0 + tid], a.meta->len[b0 + tid], page, r);
        s_slot[tid] = page;
        s_len[tid] = r;
    }
    __syncthreads();
    if (!s_flag) {
        if (producer && lane == 0)
            for (int i2 = 0; i2 < n_issued; ++i2) mbar_wait_bounded(&full[i2], 0, nullptr);
        return;
    }
    (void)mbar_try_wait(&bar_x, 0);
    // rows past the batch are zero
    for (int e = tid; e < (BT - nb) * XS; e += kMmaThreads) sX[static_cast<size_t>(nb) * XS + e] = 0.0f;
    __syncthreads();

    unsigned long long best[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) best[nt][0] = best[nt][1] = 0ull;

    const int g = lane >> 2, t = lane & 3;
    // Global inputs of one output element's epilogue (row scale, bias, residual value).
    // A warp loads all of them for its elements before its first store: a load placed
    // after a store to memory it might alias waits for that store, one L2 round trip
    // per element.
    struct EpiIn {
        float s, bias, prev;
    };
    auto load_in = [&](int n, int b) {
        EpiIn v{1.0f, 0.0f, 0.0f};
        if (!F32W) v.s = a.scale[n];
        if (EPI != EPI_HEAD && a.bias != nullptr) v.bias = a.bias[n];
        if (EPI == EPI_RESID) v.prev = a.out[static_cast<long long>(b0 + b) * a.out_ld + n];
        return v;
    };
    // epilogue of one output element
    // (nt, e: the argmax accumulator of column b = 8 nt + 2 t + e, compile-time at every
    // call; nt < 0 folds into the CTA's shared keys instead)
    auto finish = [&](int n, int b, float y, const EpiIn& in, int nt, int e) {
        if (!F32W) y = __fmul_rn(y, in.s);
        if (EPI != EPI_HEAD && a.bias != nullptr) y = __fadd_rn(y, in.bias);
        const int gb = b0 + b;
        if (EPI == EPI_STORE) {
            a.out[static_cast<long long>(gb) * a.out_ld + n] = y;
        } else if (EPI == EPI_RESID) {
            a.out[static_cast<long long>(gb) * a.out_ld + n] = __fadd_rn(in.prev, y);
        } else if (EPI == EPI_GELU) {
            a.out[static_cast<long long>(gb) * a.out_ld + n] = gelu_tanh_f(y);
        } else if (EPI == EPI_QKV) {
            const int sec = n < a.d ? 0 : (n < a.d + a.kvd ? 1 : 2);
            const int within = n - (sec == 0 ? 0 : (sec == 1 ? a.d : a.d + a.kvd));
            const int hh = within >> 6, i = within & 63;
            if (sec == 0) {
                a.out[static_cast<long long>(gb) * a.out_ld + within] = y;
            } else {
                float* cache = (sec == 1) ? a.kc : a.vc;
                cache[kv_page_off(a.kv, s_slot[b], hh, s_len[b]) + i] = y;
            }
        } else if (EPI == EPI_HEAD) {
            if (a.out != nullptr) a.out[static_cast<long long>(gb) * a.out_ld + n] = y;
            const unsigned long long key = argmax_key(y, n);
            if (nt < 0)
                atomicMax(&s_key[b], key);   // split-K reduction: column b of this warp's rows
            else
                best[nt][e] = key > best[nt][e] ? key : best[nt][e];
        }
    };

    if (producer) {
        if (lane == 0) {
            for (int it = n_issued; it < n_items; ++it) {
                const int stage = it % NS;
                if (!mbar_wait_bounded(&empty[stage], static_cast<uint32_t>(it / NS - 1) & 1u, a.err)) break;
                issue(it);
                n_issued = it + 1;
            }
            for (int i2 = max(0, n_issued - NS); i2 < n_issued; ++i2)
                mbar_wait_bounded(&full[i2 % NS], static_cast<uint32_t>(i2 / NS) & 1u, nullptr);
        }
    } else {
        float acc[2][NT][4];
        for (int it = 0; it < n_items; ++it) {
            const int stage = it % NS;
            const uint32_t phase = static_cast<uint32_t>(it / NS) & 1u;
            int ok = 1;
            if (lane == 0) ok = mbar_wait_bounded(&full[stage], phase, a.err) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (lane != 0) (void)mbar_try_wait(&full[stage], phase);
            const int jb = c0 + (it / nkc) * cps;
            const int c = it % nkc;
            if (c == 0) {
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.0f;
            }
            const unsigned char* st = ring + static_cast<size_t>(stage) * SB;
            // 32-column groups of this stage (slices and K are multiples of 32); the group
            // body is unrolled, the group loop is not, so the code stays in the
            // instruction cache
            constexpr int QPB = BOXK / 32;
            const int ngrp = min(KC, klen - c * KC) / 32;
#pragma unroll 1
            for (int grp = 0; grp < ngrp; ++grp) {
                const int bx = grp / QPB, q = grp - bx * QPB;
                const unsigned char* box = st + bx * kMmaBoxBytes;
                {
                    const int kl = c * KC + grp * 32;   // column within the slice
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        // four physical columns kl + pcol .. +3 serve MMA steps 2h and 2h + 1
                        const int pcol = mma_pcol<WT>(t, h);
                        const int woff = (q * 32 + pcol) * ELT;
                        float4 wv[2][2];
#pragma unroll
                        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                            for (int rr = 0; rr < 2; ++rr)
                                wv[mt][rr] = load_w4<WT>(box, 32 * warp + 16 * mt + g + 8 * rr, woff);
                        uint4 xh[NT], xl[NT];   // TF32 split of the activations
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const size_t o = static_cast<size_t>(nt * 8 + g) * XS + kl + pcol;
                            const float4 xv = *reinterpret_cast<const float4*>(sX + o);
                            xh[nt] = make_uint4(tf32_of(xv.x), tf32_of(xv.y), tf32_of(xv.z), tf32_of(xv.w));
                            xl[nt] = make_uint4(tf32_of(xv.x - __uint_as_float(xh[nt].x)),
                                                tf32_of(xv.y - __uint_as_float(xh[nt].y)),
                                                tf32_of(xv.z - __uint_as_float(xh[nt].z)),
                                                tf32_of(xv.w - __uint_as_float(xh[nt].w)));
                        }
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            uint32_t ahi[2][4], alo[2][4];
#pragma unroll
                            for (int mt = 0; mt < 2; ++mt) {
                                const float w0 = j ? wv[mt][0].z : wv[mt][0].x;   // row g,   logical k = t
                                const float w1 = j ? wv[mt][1].z : wv[mt][1].x;   // row g+8, logical k = t
                                const float w2 = j ? wv[mt][0].w : wv[mt][0].y;   // row g,   logical k = t + 4
                                const float w3 = j ? wv[mt][1].w : wv[mt][1].y;   // row g+8, logical k = t + 4
                                if (F32W) {
                                    ahi[mt][0] = tf32_of(w0);
                                    ahi[mt][1] = tf32_of(w1);
                                    ahi[mt][2] = tf32_of(w2);
                                    ahi[mt][3] = tf32_of(w3);
                                    alo[mt][0] = tf32_of(w0 - __uint_as_float(ahi[mt][0]));
                                    alo[mt][1] = tf32_of(w1 - __uint_as_float(ahi[mt][1]));
                                    alo[mt][2] = tf32_of(w2 - __uint_as_float(ahi[mt][2]));
                                    alo[mt][3] = tf32_of(w3 - __uint_as_float(ahi[mt][3]));
                                } else {
                                    // integers below 2^8 are exact TF32 values
                                    ahi[mt][0] = __float_as_uint(w0);
                                    ahi[mt][1] = __float_as_uint(w1);
                                    ahi[mt][2] = __float_as_uint(w2);
                                    ahi[mt][3] = __float_as_uint(w3);
                                }
                            }
                            // small terms first; the 2 x NT accumulators interleave so that
                            // consecutive MMAs are independent
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                                for (int mt = 0; mt < 2; ++mt)
                                    mma_tf32(acc[mt][nt], ahi[mt], j ? xl[nt].z : xl[nt].x, j ? xl[nt].w : xl[nt].y);
                            if (F32W) {
#pragma unroll
                                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                                    for (int mt = 0; mt < 2; ++mt)
                                        mma_tf32(acc[mt][nt], alo[mt], j ? xh[nt].z : xh[nt].x, j ? xh[nt].w : xh[nt].y);
                            }
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                                for (int mt = 0; mt < 2; ++mt)
                                    mma_tf32(acc[mt][nt], ahi[mt], j ? xh[nt].z : xh[nt].x, j ? xh[nt].w : xh[nt].y);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (c != nkc - 1) continue;
            // ---- block done: epilogue directly, or through the split-K reduction ----
            // C fragment: e = 0,1 -> row g, columns 2t, 2t+1; e = 2,3 -> row g + 8
            if (A.n_ks == 1) {
                EpiIn in[2][NT][4];
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int n = jb * kMmaBlockRows + 32 * warp + 16 * mt + g + 8 * (e >> 1);
                            const int b = nt * 8 + 2 * t + (e & 1);
                            if (b < nb && n < a.N) in[mt][nt][e] = load_in(n, b);
                        }
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int n = jb * kMmaBlockRows + 32 * warp + 16 * mt + g + 8 * (e >> 1);
                            const int b = nt * 8 + 2 * t + (e & 1);
                            if (b < nb && n < a.N) finish(n, b, acc[mt][nt][e], in[mt][nt][e], nt, e & 1);
                        }
            } else {
                float* tile = reinterpret_cast<float*>(A.part) +
                              ((static_cast<long long>(jb) * n_by + by) * A.n_ks + ks) * (kMmaBlockRows * BT);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int rr = 0; rr < 2; ++rr) {
                            const int lr = 32 * warp + 16 * mt + g + 8 * rr;
                            *reinterpret_cast<float2*>(tile + lr * BT + nt * 8 + 2 * t) =
                                make_float2(acc[mt][nt][2 * rr], acc[mt][nt][2 * rr + 1]);
                        }
                // each warp's 32 rows are reduced on their own: the last of the n_ks
                // warps that own them (arrival count, no waiting) sums the slices
                __threadfence();
                __syncwarp();
                int* cw = A.cnt + (static_cast<long long>(jb) * n_by + by) * kMmaConsumerWarps + warp;
                int last = 0;
                if (lane == 0) last = (atomicAdd(cw, 1) == A.n_ks - 1);
                last = __shfl_sync(0xffffffffu, last, 0);
                if (last) {
                    __threadfence();
                    // this warp's rows are 32 x BT contiguous floats in every slice's
                    // tile; lane takes float4 j at lane + 32 j, slices summed in order
                    constexpr int V = BT / 4;
                    constexpr int U = 4;   // slices in flight
                    const float4* wb = reinterpret_cast<const float4*>(
                        reinterpret_cast<const float*>(A.part) +
                        (static_cast<long long>(jb) * n_by + by) * A.n_ks * (kMmaBlockRows * BT) + 32 * warp * BT);
                    const long long sstride = kMmaBlockRows * BT / 4;
                    float4 sum[V];
#pragma unroll
                    for (int j = 0; j < V; ++j) sum[j] = make_float4(0.f, 0.f, 0.f, 0.f);
                    int i = 0;
                    for (; i + U <= A.n_ks; i += U) {
                        float4 v[U][V];
#pragma unroll
                        for (int u = 0; u < U; ++u)
#pragma unroll
                            for (int j = 0; j < V; ++j) v[u][j] = __ldcg(wb + (i + u) * sstride + lane + 32 * j);
#pragma unroll
                        for (int u = 0; u < U; ++u)
#pragma unroll
                            for (int j = 0; j < V; ++j) {
                                sum[j].x += v[u][j].x;
                                sum[j].y += v[u][j].y;
                                sum[j].z += v[u][j].z;
                                sum[j].w += v[u][j].w;
                            }
                    }
                    for (; i < A.n_ks; ++i) {
#pragma unroll
                        for (int j = 0; j < V; ++j) {
                            const float4 v = __ldcg(wb + i * sstride + lane + 32 * j);
                            sum[j].x += v.x;
                            sum[j].y += v.y;
                            sum[j].z += v.z;
                            sum[j].w += v.w;
                        }
                    }
                    EpiIn in[V][4];
#pragma unroll
                    for (int j = 0; j < V; ++j) {
                        const int e0 = (lane + 32 * j) * 4;
                        const int n = jb * kMmaBlockRows + 32 * warp + e0 / BT;
                        const int bc = e0 % BT;
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            if (n < a.N && bc + u < nb) in[j][u] = load_in(n, bc + u);
                    }
#pragma unroll
                    for (int j = 0; j < V; ++j) {
                        const int e0 = (lane + 32 * j) * 4;
                        const int n = jb * kMmaBlockRows + 32 * warp + e0 / BT;
                        const int bc = e0 % BT;
                        if (n < a.N) {
                            if (bc < nb) finish(n, bc, sum[j].x, in[j][0], -1, 0);
                            if (bc + 1 < nb) finish(n, bc + 1, sum[j].y, in[j][1], -1, 0);
                            if (bc + 2 < nb) finish(n, bc + 2, sum[j].z, in[j][2], -1, 0);
                            if (bc + 3 < nb) finish(n, bc + 3, sum[j].w, in[j][3], -1, 0);
                        }
                    }
                    if (lane == 0) *cw = 0;
                }
            }
        }
    }

    if (EPI == EPI_HEAD) {
        __syncthreads();
        if (!producer) {
            // fold over the 8 row groups g that share a column pair
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    unsigned long long v = best[nt][e];
#pragma unroll
                    for (int off = 4; off < 32; off <<= 1) {
                        const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, off);
                        v = o > v ? o : v;
                    }
                    const int b = nt * 8 + 2 * (lane & 3) + e;
                    if (lane < 4 && b < nb && v != 0ull) atomicMax(&s_key[b], v);
                }
        }
        __syncthreads();
        if (tid < nb && s_key[tid] != 0ull) atomicMax(&a.keys[b0 + tid], s_key[tid]);
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            const int total = gridDim.x;
            s_last = (atomicAdd(a.counter, 1) == total - 1);
        }
        __syncthreads();
        if (s_last) {
            __threadfence();
            for (int b = tid; b < a.B; b += kMmaThreads) {
                const unsigned long long k = atomicExch(&a.keys[b], 0ull);
                const int idx = (k == 0ull) ? 0 : argmax_key_index(k);
                if (a.argmax_out) a.argmax_out[b] = idx;
                if (a.last_tok) a.last_tok[a.meta->slot[b]] = idx;
            }
            if (tid == 0) *a.counter = 0;
        }
    }
}

// ---------------------------------------------------------------- launch planning

constexpr int kMmaMaxBT = 32;                  // batch columns per CTA at most
constexpr size_t kMmaXBudget = 96 * 1024;      // activation slice bytes at most

// K split of one projection. It depends only on the matrix shape, the weight type and
// the SM count -- never on the batch -- so every output element is summed in the same
// order at every batch size.
struct MmaPlan {
    int n_blocks;   // 128-row blocks
    int n_ks;       // K slices
    int ksl;        // K elements per slice
    int nbx;        // 128-byte boxes per pipeline stage (TF32 kernel)
    bool ok;
};

inline MmaPlan mma_plan(int N, int K, int elt, int num_sms) {
    MmaPlan p{};
    // int8 weights stream 128 columns (16 KB) per stage: finer K slices, so that the
    // 2xTF32 work of a slice spreads over every SM
    p.nbx = elt == 1 ? 1 : 2;
    const int KC = p.nbx * 128 / elt;
    const int pad = elt == 4 ? 4 : 16;
    p.n_blocks = (N + kMmaBlockRows - 1) / kMmaBlockRows;
    if (K % 32 != 0 || N <= 0) return p;
    const int kchunks = (K + KC - 1) / KC;
    // one wave: n_blocks x n_ks CTAs within the SM count (the f32 activation slices and the
    // split TF32 products make this kernel's CTAs heavier than the int8 kernel's, and fewer
    // slices measured slower on B200 for the C2 and C5 shapes)
    int n_ks = std::max(1, std::min(kchunks, num_sms / std::max(1, p.n_blocks)));
    auto slice_len = [&](int nks) { return std::min(((kchunks + nks - 1) / nks) * KC, K); };
    auto xbytes = [&](int ksl) { return size_t(kMmaMaxBT) * (ksl + pad) * 4; };
    while (xbytes(slice_len(n_ks)) > kMmaXBudget && n_ks < kchunks) ++n_ks;
    p.ksl = slice_len(n_ks);
    p.n_ks = (K + p.ksl - 1) / p.ksl;
    p.ok = xbytes(p.ksl) <= kMmaXBudget;
    return p;
}

// Scratch of one launch with batch B: partial tiles (bytes) and arrival counters.
inline size_t mma_part_bytes(const MmaPlan& p, int B) {
    const int gy = (B + kMmaMaxBT - 1) / kMmaMaxBT;
    return p.n_ks > 1 ? size_t(p.n_blocks) * gy * p.n_ks * kMmaBlockRows * kMmaMaxBT * 4 : 0;
}
inline int mma_counters(const MmaPlan& p, int B) {
    return p.n_blocks * ((B + kMmaMaxBT - 1) / kMmaMaxBT) * kMmaConsumerWarps;
}

template <typename WT, int EPI>
cudaError_t proj_mma_launch(int num_sms, const CUtensorMap& map, void* part, size_t part_bytes, int* cnt,
                            int cnt_len, const GemvArgs& g, cudaStream_t st);

template <int PRO>
cudaError_t rowprep_launch(const GemvArgs& g, float* out, cudaStream_t st);

#ifdef DEC_MMA_DEFINE

template <int BT, typename WT, int EPI, int NBX>
cudaError_t proj_mma_launch_bt(int num_sms, MmaArgs A, int n_blocks, cudaStream_t st) {
    auto kern = k_proj_mma<BT, WT, EPI, NBX>;
    constexpr int SB = kMmaBoxBytes * NBX;
    const size_t xbytes = size_t(BT) * (A.ksl + mma_xpad<WT>()) * 4;
    const size_t avail = size_t(227 * 1024) - 1024 - 1024 - xbytes;
    const int ns_max = int(std::min<size_t>(kMmaMaxStagesTF, avail / SB));
    if (ns_max < 2) return cudaErrorNotSupported;
    thread_local int attr_dev = -1;   // attributes are per device; set again when it changes
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (attr_dev != dev) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024 - 1024);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        attr_dev = dev;
    }
    // the ring holds no more stages than a CTA streams (room for the next kernel's CTAs)
    const int gy = (A.g.B + BT - 1) / BT;
    A.n_by = gy;
    const int stage_k = NBX * 128 / int(sizeof(WT));
    const int nkc = (A.ksl + stage_k - 1) / stage_k;
    int occ = 0, cps = 1, NS = ns_max;
    for (int pass = 0; pass < 2; ++pass) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kMmaThreads,
                                                          1024 + size_t(pass == 0 ? 2 : NS) * SB + xbytes);
        if (e != cudaSuccess) return e;
        const int slots = std::max(1, num_sms * std::max(1, occ) / gy);
        cps = std::max(1, std::min(n_blocks, slots / A.n_ks));
        NS = std::min(ns_max, std::max(2, ((n_blocks + cps - 1) / cps) * nkc));
    }
    const size_t smem = 1024 + size_t(NS) * SB + xbytes;
    // one wave at the final ring depth
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kMmaThreads, smem);
    if (e != cudaSuccess) return e;
    cps = std::max(1, std::min(cps, std::max(1, num_sms * std::max(1, occ) / gy) / A.n_ks));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cps * A.n_ks * gy);
    cfg.blockDim = dim3(kMmaThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, A, NS);
}

template <typename WT, int EPI>
cudaError_t proj_mma_launch(int num_sms, const CUtensorMap& map, void* part, size_t part_bytes, int* cnt,
                            int cnt_len, const GemvArgs& g, cudaStream_t st) {
    if (g.B < 1) return cudaErrorNotSupported;
    const MmaPlan p = mma_plan(g.N, g.K, int(sizeof(WT)), num_sms);
    if (!p.ok) return cudaErrorNotSupported;
    if (p.n_ks > 1 && (mma_part_bytes(p, g.B) > part_bytes || mma_counters(p, g.B) > cnt_len))
        return cudaErrorNotSupported;
    int bt = 8;
    while (bt < g.B && bt < kMmaMaxBT) bt <<= 1;
    MmaArgs A;
    A.tmap = map;
    A.part = part;
    A.cnt = cnt;
    A.n_ks = p.n_ks;
    A.ksl = p.ksl;
    A.n_by = 1;
    A.g = g;
    if (p.nbx == 1) {
        switch (bt) {
            case 8: return proj_mma_launch_bt<8, WT, EPI, 1>(num_sms, A, p.n_blocks, st);
            case 16: return proj_mma_launch_bt<16, WT, EPI, 1>(num_sms, A, p.n_blocks, st);
            default: return proj_mma_launch_bt<32, WT, EPI, 1>(num_sms, A, p.n_blocks, st);
        }
    }
    switch (bt) {
        case 8: return proj_mma_launch_bt<8, WT, EPI, 2>(num_sms, A, p.n_blocks, st);
        case 16: return proj_mma_launch_bt<16, WT, EPI, 2>(num_sms, A, p.n_blocks, st);
        default: return proj_mma_launch_bt<32, WT, EPI, 2>(num_sms, A, p.n_blocks, st);
    }
}

template <int PRO>
cudaError_t rowprep_launch(const GemvArgs& g, float* out, cudaStream_t st) {
    if (g.K > kRowprepMaxK || g.K % 4 != 0) return cudaErrorNotSupported;
    thread_local int attr_dev = -1;
    const cudaError_t e = prefer_max_shared_once(k_rowprep<PRO>, attr_dev);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g.B);
    cfg.blockDim = dim3(kRowprepThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_rowprep<PRO>, g.x, g.x_ld, g.norm_w, g.norm_b, g.eps, g.K, out);
}

#define DEC_MMA_INSTANTIATE(WT, EPI)                                                                   \
    template cudaError_t proj_mma_launch<WT, EPI>(int, const CUtensorMap&, void*, size_t, int*, int, \
                                                  const GemvArgs&, cudaStream_t);
#define DEC_ROWPREP_INSTANTIATE(PRO) template cudaError_t rowprep_launch<PRO>(const GemvArgs&, float*, cudaStream_t);

#endif  // DEC_MMA_DEFINE

}  // namespace dec
