// Tensor-core projections for W8A8 layers (int8 per-row weights, int8 activation rows
// with one scale per row), for batches of 8 to 64 streams: mma.sync m16n8k32 on int8
// operands with exact int32 accumulation. The activation rows come from k_rowprep_i8,
// the per-row symmetric quantiser with ties to even (franken_ocr decoder_qwen2.rs,
// quantize_row_i8_te), computed with the CUDA-core kernel's arithmetic and reduction
// order; the int32 sums are exact, so y = float(acc) * (a_b * s_n) + bias is bit-identical
// to the CUDA-core dp4a kernel's (decoder_qwen2.rs, gemv_i8_bias_prequant).
//
// Decomposition, pipeline and split-K reduction follow the TF32 kernel (proj_mma.cuh):
// 128-row weight blocks streamed by one producer warp with 2-D TMA loads (no multicast)
// into a ring of 32 KB stages, K slices owned by CTA groups, four consumer warps of 32
// rows x all batch columns. Partial tiles are stored in fragment order (each lane's
// float4 / int4 of every (m16, n8) tile contiguous across the warp), so the last of the
// n_ks warps that own a 32-row group reads back exactly its own fragments, sums the slices
// in slice order and runs the same epilogue as the unsplit case.
//
// Row maps: the epilogue needs rows i and i + 32 of a head together (NEOX RoPE) or the
// gate and up rows of one output together (SwiGLU). The weights of those projections are
// stored permuted for this kernel so that the pair lands in rows g and g + 8 of one m16
// tile -- the two rows a thread holds in its accumulator fragment:
//   MAP_ROPE: in each 64-row head block, physical row 16 m + l holds logical row
//             8 m + l (l < 8) or 32 + 8 m + (l - 8) (l >= 8);
//   MAP_DUAL: physical row 16 j + l holds gate row 8 j + l (l < 8) or up row 8 j + l - 8.
#pragma once

#include "proj_mma.cuh"

namespace dec {

constexpr int kI8KC = kMmaBoxesPerStage * 128;   // K elements per stage (256)
constexpr int kI8XPad = 16;                      // activation row padding (bytes)
constexpr int kI8MaxBT = 64;                     // batch columns per CTA at most

struct I8MmaArgs {
    CUtensorMap tmap;        // int8 weights [N_phys, K]: box {128 bytes, 128 rows}, 128-byte swizzle
    void* part;              // split-K partial tiles (fragment order)
    int* cnt;                // split-K arrival counts per (row block, batch tile, warp), zero between launches
    int n_ks;                // K slices
    int ksl;                 // K elements per slice (a multiple of 256, or K)
    int n_rows;              // physical weight rows (2 N for MAP_DUAL)
    int n_by;                // batch tiles (the fastest-varying CTA index)
    const int8_t* xq;        // [B, K] quantised activations
    const float* xs;         // [B] activation scales
    GemvArgs g;              // shapes and epilogue arguments
};

__device__ __forceinline__ void mma_s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four int8 weights at byte `off` (multiple of 4) of local row `lr` of a swizzled box.
__device__ __forceinline__ uint32_t load_w_s8x4(const unsigned char* box, int lr, int off) {
    return *reinterpret_cast<const uint32_t*>(box + lr * 128 + ((((off >> 4) ^ (lr & 7))) << 4) + (off & 15));
}

// Logical row of physical row p under a row map.
template <int MAP>
__host__ __device__ __forceinline__ int i8_logical_row(int p) {
    if (MAP == MAP_ROPE) {
        const int w = p & 63, m = w >> 4, l = w & 15;
        return (p & ~63) + (l < 8 ? 8 * m + l : 32 + 8 * m + (l - 8));
    }
    if (MAP == MAP_DUAL) return ((p >> 4) << 3) + (p & 7);   // output row (gate if (p & 8) == 0)
    return p;
}

// Per-row int8 quantisation (optionally after RMSNorm or LayerNorm), one warp per row,
// with the arithmetic and reduction order of the CUDA-core kernel's prologue so that both
// paths produce the same codes and scales.
template <int PRO>
__global__ void __launch_bounds__(128) k_rowprep_i8(const float* __restrict__ x, int x_ld,
                                                    const float* __restrict__ gw, const float* __restrict__ gb,
                                                    float eps, int K, int B, int8_t* __restrict__ xq,
                                                    float* __restrict__ xs) {
    pdl_launch_dependents();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.x * 4 + (threadIdx.x >> 5);
    if (b >= B) return;
    const float4* xr = reinterpret_cast<const float4*>(x + static_cast<long long>(b) * x_ld);
    const float4* g4 = reinterpret_cast<const float4*>(gw);
    const float4* be4 = reinterpret_cast<const float4*>(gb);
    const int K4 = K >> 2;
    float mu = 0.0f, rstd = 1.0f;
    if (PRO == PRO_LN) {
        float sum = 0.0f;
        for (int k = lane; k < K4; k += 32) {
            const float4 v = xr[k];
            sum += (v.x + v.y) + (v.z + v.w);
        }
        mu = warp_sum(sum) / static_cast<float>(K);
        float var = 0.0f;
        for (int k = lane; k < K4; k += 32) {
            const float4 v = xr[k];
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
        for (int k = lane; k < K4; k += 32) {
            const float4 v = xr[k];
            ss = fmaf(v.x, v.x, ss);
            ss = fmaf(v.y, v.y, ss);
            ss = fmaf(v.z, v.z, ss);
            ss = fmaf(v.w, v.w, ss);
        }
        ss = warp_sum(ss) / static_cast<float>(K);
        rstd = 1.0f / sqrtf(ss + eps);
    }
    auto normed = [&](int k) {
        const float4 v = xr[k];
        float4 g = make_float4(1.f, 1.f, 1.f, 1.f), be = make_float4(0.f, 0.f, 0.f, 0.f);
        if (PRO != PRO_NONE) g = __ldg(g4 + k);
        if (PRO == PRO_LN) be = __ldg(be4 + k);
        return make_float4(norm_value(PRO, v.x, mu, rstd, g.x, be.x), norm_value(PRO, v.y, mu, rstd, g.y, be.y),
                           norm_value(PRO, v.z, mu, rstd, g.z, be.z), norm_value(PRO, v.w, mu, rstd, g.w, be.w));
    };
    float amax = 0.0f;
    for (int k = lane; k < K4; k += 32) {
        const float4 y = normed(k);
        amax = fmaxf(amax, fabsf(y.x));
        amax = fmaxf(amax, fabsf(y.y));
        amax = fmaxf(amax, fabsf(y.z));
        amax = fmaxf(amax, fabsf(y.w));
    }
    amax = warp_max(amax);
    const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
    uint32_t* q = reinterpret_cast<uint32_t*>(xq + static_cast<long long>(b) * K);
    for (int k = lane; k < K4; k += 32) {
        const float4 y = normed(k);
        q[k] = (static_cast<uint32_t>(quant_i8(y.x, inv)) & 0xffu) |
               ((static_cast<uint32_t>(quant_i8(y.y, inv)) & 0xffu) << 8) |
               ((static_cast<uint32_t>(quant_i8(y.z, inv)) & 0xffu) << 16) |
               ((static_cast<uint32_t>(quant_i8(y.w, inv)) & 0xffu) << 24);
    }
    if (lane == 0) xs[b] = __fdiv_rn(amax, 127.0f);
}

template <int BT, int EPI, int MAP>
__global__ void __launch_bounds__(kMmaThreads, 1) k_proj_i8mma(const __grid_constant__ I8MmaArgs A, int NS) {
    const GemvArgs& a = A.g;
    constexpr int NT = BT / 8;
    constexpr int QPB = 128 / 32;   // 32-column groups per box
    static_assert(BT % 8 == 0, "tile");

    extern __shared__ unsigned char i8_smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(i8_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    unsigned char* ring = smem;
    const int XSB = A.ksl + kI8XPad;   // activation row (bytes)
    int8_t* sX = reinterpret_cast<int8_t*>(smem + static_cast<size_t>(NS) * kMmaStageBytes);
    __shared__ __align__(8) uint64_t full[kMmaMaxStages];
    __shared__ __align__(8) uint64_t empty[kMmaMaxStages];
    __shared__ __align__(8) uint64_t bar_x;
    __shared__ float s_rs[BT];   // activation scales a_b
    __shared__ int s_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool producer = warp == kMmaConsumerWarps;
    // batch tile fastest, so that the tiles of one weight block read it together
    const int n_by = A.n_by;
    const int by = blockIdx.x % n_by, b0 = by * BT;
    const int nb = min(BT, a.B - b0);
    const int n_blocks = (A.n_rows + kMmaBlockRows - 1) / kMmaBlockRows;
    const int rest = blockIdx.x / n_by;
    const int ks = rest % A.n_ks;
    const int cps = gridDim.x / (A.n_ks * n_by);
    const int c0 = rest / A.n_ks;
    const int kstart = ks * A.ksl;
    const int klen = min(A.ksl, a.K - kstart);
    const int nkc = (klen + kI8KC - 1) / kI8KC;
    const int my_blocks = (c0 < n_blocks && cps > 0) ? (n_blocks - 1 - c0) / cps + 1 : 0;
    const int n_items = my_blocks * nkc;

    auto issue = [&](int it) {
        const int jb = c0 + (it / nkc) * cps;
        const int c = it % nkc;
        const int stage = it % NS;
        unsigned char* dst = ring + static_cast<size_t>(stage) * kMmaStageBytes;
        mbar_arrive_expect_tx(&full[stage], kMmaStageBytes);
#pragma unroll
        for (int bx = 0; bx < kMmaBoxesPerStage; ++bx)
            tma_load_2d(dst + bx * kMmaBoxBytes, &A.tmap, kstart + c * kI8KC + bx * 128, jb * kMmaBlockRows,
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

    // ---- activation slice: one bulk copy per row ----
    if (producer && lane == 0) {
        mbar_arrive_expect_tx(&bar_x, static_cast<uint32_t>(klen) * nb);
        for (int b = 0; b < nb; ++b)
            bulk_g2s(sX + static_cast<size_t>(b) * XSB, A.xq + static_cast<long long>(b0 + b) * a.K + kstart,
                     static_cast<uint32_t>(klen), &bar_x);
        s_flag = mbar_wait_bounded(&bar_x, 0, a.err) ? 1 : 0;
    }
    if (tid < BT) s_rs[tid] = tid < nb ? A.xs[b0 + tid] : 0.0f;
    // rows past the batch are zero
    for (int e = tid; e < (BT - nb) * XSB; e += kMmaThreads) sX[static_cast<size_t>(nb) * XSB + e] = 0;
    __syncthreads();
    if (!s_flag) {
        if (producer && lane == 0)
            for (int i2 = 0; i2 < n_issued; ++i2) mbar_wait_bounded(&full[i2], 0, nullptr);
        return;
    }
    (void)mbar_try_wait(&bar_x, 0);

    const int g = lane >> 2, t = lane & 3;

    // epilogue of one (m16, n8) fragment of exact sums: v[0], v[1] row p0 cols 2t, 2t+1;
    // v[2], v[3] row p0 + 8
    auto finish_frag = [&](int jb, int mt, int nt, const int (&v)[4]) {
        const int p0 = jb * kMmaBlockRows + 32 * warp + 16 * mt + g;   // physical rows p0, p0 + 8
        float y[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int p = p0 + 8 * (e >> 1);
            const int b = nt * 8 + 2 * t + (e & 1);
            const int n = i8_logical_row<MAP>(p);
            const float* sc = (MAP == MAP_DUAL && (e >> 1)) ? a.scale2 : a.scale;
            const bool live = p < A.n_rows && b < nb;
            y[e] = __fmul_rn(static_cast<float>(v[e]), __fmul_rn(s_rs[b], sc[live ? n : 0]));
            if (EPI != EPI_SWIGLU && a.bias != nullptr && live) y[e] = __fadd_rn(y[e], a.bias[n]);
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int b = nt * 8 + 2 * t + e;
            if (b >= nb) continue;
            const int gb = b0 + b;
            if (EPI == EPI_SWIGLU) {
                // gate in row p0, up in row p0 + 8, both for output n
                if (p0 < A.n_rows)
                    a.out[static_cast<long long>(gb) * a.out_ld + i8_logical_row<MAP>(p0)] =
                        __fmul_rn(silu_f(y[e]), y[2 + e]);
                continue;
            }
            if (EPI == EPI_QKV && MAP == MAP_ROPE) {
                if (p0 >= A.n_rows) continue;
                const int n0 = i8_logical_row<MAP>(p0);   // i < 32; its partner is i + 32
                const int sec = n0 / a.d, within = n0 - sec * a.d;
                const int hh = within >> 6, i = within & 63;
                float v0 = y[e], v1 = y[2 + e];
                if (a.rope != nullptr && sec < 2) {
                    const float2 cs = a.rope[static_cast<long long>(a.meta->pos[gb]) * 32 + i];
                    v0 = __fsub_rn(__fmul_rn(y[e], cs.x), __fmul_rn(y[2 + e], cs.y));
                    v1 = __fadd_rn(__fmul_rn(y[e], cs.y), __fmul_rn(y[2 + e], cs.x));
                }
                if (sec == 0) {
                    a.out[static_cast<long long>(gb) * a.out_ld + within] = v0;
                    a.out[static_cast<long long>(gb) * a.out_ld + within + 32] = v1;
                } else {
                    const int slot = a.meta->slot[gb], row = a.meta->len[gb];
                    float* cache = (sec == 1) ? a.kc : a.vc;
                    float* dst = cache + slot * a.slot_stride + (static_cast<long long>(hh) * a.ld + row) * kHeadDim;
                    dst[i] = v0;
                    dst[i + 32] = v1;
                }
                continue;
            }
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int p = p0 + 8 * r;
                if (p >= A.n_rows) continue;
                const int n = i8_logical_row<MAP>(p);
                const float yv = y[2 * r + e];
                if (EPI == EPI_STORE) {
                    a.out[static_cast<long long>(gb) * a.out_ld + n] = yv;
                } else if (EPI == EPI_RESID) {
                    float* q = a.out + static_cast<long long>(gb) * a.out_ld + n;
                    *q = __fadd_rn(*q, yv);
                }
            }
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
        return;
    }

    int acc[2][NT][4];
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
                    for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0;
        }
        const unsigned char* st = ring + static_cast<size_t>(stage) * kMmaStageBytes;
        const int ngrp = min(kI8KC, klen - c * kI8KC) / 32;
#pragma unroll 1
        for (int grp = 0; grp < ngrp; ++grp) {
            const int bx = grp / QPB, q = grp - bx * QPB;
            const unsigned char* box = st + bx * kMmaBoxBytes;
            const int kl = c * kI8KC + grp * 32;   // column within the slice
            uint32_t af[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const int lr = 32 * warp + 16 * mt + g;
                af[mt][0] = load_w_s8x4(box, lr, q * 32 + 4 * t);
                af[mt][1] = load_w_s8x4(box, lr + 8, q * 32 + 4 * t);
                af[mt][2] = load_w_s8x4(box, lr, q * 32 + 16 + 4 * t);
                af[mt][3] = load_w_s8x4(box, lr + 8, q * 32 + 16 + 4 * t);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int8_t* xr = sX + static_cast<size_t>(nt * 8 + g) * XSB + kl + 4 * t;
                const uint32_t bq0 = *reinterpret_cast<const uint32_t*>(xr);
                const uint32_t bq1 = *reinterpret_cast<const uint32_t*>(xr + 16);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) mma_s8(acc[mt][nt], af[mt], bq0, bq1);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
        if (c != nkc - 1) continue;

        // ---- block done ----
        if (A.n_ks == 1) {
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) finish_frag(jb, mt, nt, acc[mt][nt]);
            continue;
        }
        // fragment-order tile of this warp: vector (mt, nt) of lane at ((mt * NT + nt) * 32 + lane)
        constexpr int WV = 2 * NT * 32;   // 16-byte vectors per warp per slice
        const long long tile_base = ((static_cast<long long>(jb) * n_by + by) * A.n_ks) * (kMmaConsumerWarps * WV);
        int4* mine = reinterpret_cast<int4*>(A.part) + tile_base + static_cast<long long>(ks) * (kMmaConsumerWarps * WV) +
                     warp * WV;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                mine[(mt * NT + nt) * 32 + lane] = make_int4(acc[mt][nt][0], acc[mt][nt][1], acc[mt][nt][2], acc[mt][nt][3]);
        __threadfence();
        __syncwarp();
        int* cw = A.cnt + (static_cast<long long>(jb) * n_by + by) * kMmaConsumerWarps + warp;
        int last = 0;
        if (lane == 0) last = (atomicAdd(cw, 1) == A.n_ks - 1);
        last = __shfl_sync(0xffffffffu, last, 0);
        if (!last) continue;
        __threadfence();
        // sum the slices (exact integer sums), U slices in flight
        constexpr int U = (2 * NT) >= 16 ? 1 : 16 / (2 * NT);
        const int4* src = reinterpret_cast<const int4*>(A.part) + tile_base + warp * WV + lane;
        int sum[2][NT][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) sum[mt][nt][e] = 0;
        int i = 0;
        for (; i + U <= A.n_ks; i += U) {
            int4 v[U][2][NT];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        v[u][mt][nt] = __ldcg(src + static_cast<long long>(i + u) * (kMmaConsumerWarps * WV) +
                                              (mt * NT + nt) * 32);
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        sum[mt][nt][0] += v[u][mt][nt].x;
                        sum[mt][nt][1] += v[u][mt][nt].y;
                        sum[mt][nt][2] += v[u][mt][nt].z;
                        sum[mt][nt][3] += v[u][mt][nt].w;
                    }
        }
        for (; i < A.n_ks; ++i) {
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int4 v = __ldcg(src + static_cast<long long>(i) * (kMmaConsumerWarps * WV) + (mt * NT + nt) * 32);
                    sum[mt][nt][0] += v.x;
                    sum[mt][nt][1] += v.y;
                    sum[mt][nt][2] += v.z;
                    sum[mt][nt][3] += v.w;
                }
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) finish_frag(jb, mt, nt, sum[mt][nt]);
        if (lane == 0) *cw = 0;
    }
}

// Weight rows in the order the row maps expect (run once, when the weights are loaded):
// dst row p = src row i8_logical_row(p); for MAP_DUAL rows with (p & 8) come from src2.
template <int MAP>
__global__ void k_i8_rows_permute(int8_t* __restrict__ dst, const int8_t* __restrict__ src,
                                  const int8_t* __restrict__ src2, int n_rows, int K) {
    const int p = blockIdx.x;
    if (p >= n_rows) return;
    const int n = i8_logical_row<MAP>(p);
    const int8_t* s = (MAP == MAP_DUAL && (p & 8)) ? src2 : src;
    const uint4* from = reinterpret_cast<const uint4*>(s + static_cast<long long>(n) * K);
    uint4* to = reinterpret_cast<uint4*>(dst + static_cast<long long>(p) * K);
    for (int k = threadIdx.x; k < K / 16; k += blockDim.x) to[k] = from[k];
}

// ---------------------------------------------------------------- launch planning

// K split of one int8 projection; like mma_plan it depends on the shape and SM count
// only, never on the batch.
inline MmaPlan i8mma_plan(int n_rows, int K, int num_sms) {
    MmaPlan p{};
    p.n_blocks = (n_rows + kMmaBlockRows - 1) / kMmaBlockRows;
    if (K % 32 != 0 || n_rows <= 0) return p;
    const int kchunks = (K + kI8KC - 1) / kI8KC;
    auto xbytes = [&](int ksl) { return size_t(kI8MaxBT) * (ksl + kI8XPad); };
    int n_ks = std::max(1, std::min(std::min(kchunks, 8), num_sms / std::max(1, p.n_blocks)));
    auto slice_len = [&](int nks) { return std::min(((kchunks + nks - 1) / nks) * kI8KC, K); };
    while (xbytes(slice_len(n_ks)) > kMmaXBudget && n_ks < kchunks) ++n_ks;
    p.ksl = slice_len(n_ks);
    p.n_ks = (K + p.ksl - 1) / p.ksl;
    p.ok = xbytes(p.ksl) <= kMmaXBudget && K % 16 == 0;
    return p;
}

inline size_t i8mma_part_bytes(const MmaPlan& p, int B) {
    const int gy = (B + kI8MaxBT - 1) / kI8MaxBT;
    return p.n_ks > 1 ? size_t(p.n_blocks) * gy * p.n_ks * kMmaBlockRows * kI8MaxBT * 4 : 0;
}
inline int i8mma_counters(const MmaPlan& p, int B) {
    return p.n_blocks * ((B + kI8MaxBT - 1) / kI8MaxBT) * kMmaConsumerWarps;
}

template <int EPI, int MAP>
cudaError_t proj_i8mma_launch(int num_sms, const CUtensorMap& map, int n_rows, const int8_t* xq, const float* xs,
                              void* part, size_t part_bytes, int* cnt, int cnt_len, const GemvArgs& g,
                              cudaStream_t st);

template <int PRO>
cudaError_t rowprep_i8_launch(const GemvArgs& g, int8_t* xq, float* xs, cudaStream_t st);

// dst [n_rows, K] from src (and src2 for MAP_DUAL); K a multiple of 16.
cudaError_t i8_rows_permute(int map, int8_t* dst, const int8_t* src, const int8_t* src2, int n_rows, int K,
                            cudaStream_t st);

#ifdef DEC_I8MMA_DEFINE

cudaError_t i8_rows_permute(int map, int8_t* dst, const int8_t* src, const int8_t* src2, int n_rows, int K,
                            cudaStream_t st) {
    if (K % 16 != 0 || n_rows <= 0) return cudaErrorInvalidValue;
    if (map == MAP_ROPE) {
        if (n_rows % 64 != 0) return cudaErrorInvalidValue;
        k_i8_rows_permute<MAP_ROPE><<<n_rows, 128, 0, st>>>(dst, src, src2, n_rows, K);
    } else if (map == MAP_DUAL) {
        if (n_rows % 16 != 0) return cudaErrorInvalidValue;
        k_i8_rows_permute<MAP_DUAL><<<n_rows, 128, 0, st>>>(dst, src, src2, n_rows, K);
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

template <int BT, int EPI, int MAP>
cudaError_t proj_i8mma_launch_bt(int num_sms, I8MmaArgs A, int n_blocks, cudaStream_t st) {
    auto kern = k_proj_i8mma<BT, EPI, MAP>;
    const size_t xbytes = size_t(BT) * (A.ksl + kI8XPad);
    const size_t avail = size_t(227 * 1024) - 1024 - 1024 - xbytes;
    const int ns_max = int(std::min<size_t>(kMmaMaxStages, avail / kMmaStageBytes));
    if (ns_max < 2) return cudaErrorNotSupported;
    static int attr_dev = -1;
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
    const int stage_k = kI8KC;
    const int nkc = (A.ksl + stage_k - 1) / stage_k;
    int occ = 0, cps = 1, NS = ns_max;
    for (int pass = 0; pass < 2; ++pass) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kMmaThreads,
                                                          1024 + size_t(pass == 0 ? 2 : NS) * kMmaStageBytes + xbytes);
        if (e != cudaSuccess) return e;
        const int slots = std::max(1, num_sms * std::max(1, occ) / gy);
        cps = std::max(1, std::min(n_blocks, slots / A.n_ks));
        NS = std::min(ns_max, std::max(2, ((n_blocks + cps - 1) / cps) * nkc));
    }
    const size_t smem = 1024 + size_t(NS) * kMmaStageBytes + xbytes;
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

template <int EPI, int MAP>
cudaError_t proj_i8mma_launch(int num_sms, const CUtensorMap& map, int n_rows, const int8_t* xq, const float* xs,
                              void* part, size_t part_bytes, int* cnt, int cnt_len, const GemvArgs& g,
                              cudaStream_t st) {
    if (g.B < 1) return cudaErrorNotSupported;
    const MmaPlan p = i8mma_plan(n_rows, g.K, num_sms);
    if (!p.ok) return cudaErrorNotSupported;
    if (p.n_ks > 1 && (i8mma_part_bytes(p, g.B) > part_bytes || i8mma_counters(p, g.B) > cnt_len))
        return cudaErrorNotSupported;
    int bt = 8;
    while (bt < g.B && bt < kI8MaxBT) bt <<= 1;
    I8MmaArgs A;
    A.tmap = map;
    A.part = part;
    A.cnt = cnt;
    A.n_ks = p.n_ks;
    A.ksl = p.ksl;
    A.n_rows = n_rows;
    A.n_by = 1;
    A.xq = xq;
    A.xs = xs;
    A.g = g;
    switch (bt) {
        case 8: return proj_i8mma_launch_bt<8, EPI, MAP>(num_sms, A, p.n_blocks, st);
        case 16: return proj_i8mma_launch_bt<16, EPI, MAP>(num_sms, A, p.n_blocks, st);
        case 32: return proj_i8mma_launch_bt<32, EPI, MAP>(num_sms, A, p.n_blocks, st);
        default: return proj_i8mma_launch_bt<64, EPI, MAP>(num_sms, A, p.n_blocks, st);
    }
}

template <int PRO>
cudaError_t rowprep_i8_launch(const GemvArgs& g, int8_t* xq, float* xs, cudaStream_t st) {
    if (g.K % 16 != 0) return cudaErrorNotSupported;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((g.B + 3) / 4);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_rowprep_i8<PRO>, g.x, g.x_ld, g.norm_w, g.norm_b, g.eps, g.K, g.B, xq, xs);
}

#define DEC_I8MMA_INSTANTIATE(EPI, MAP)                                                                 \
    template cudaError_t proj_i8mma_launch<EPI, MAP>(int, const CUtensorMap&, int, const int8_t*, const float*, \
                                                     void*, size_t, int*, int, const GemvArgs&, cudaStream_t);
#define DEC_ROWPREP_I8_INSTANTIATE(PRO) \
    template cudaError_t rowprep_i8_launch<PRO>(const GemvArgs&, int8_t*, float*, cudaStream_t);

#endif  // DEC_I8MMA_DEFINE

}  // namespace dec
