// Embedding, KV-cache row copies and the cross-attention K/V precompute.
#pragma once

#include "common.cuh"

namespace dec {

// x[b] = E[token_b] (+ P[pos_b]) (cera whisper.rs `decode_step_into` step 1: token
// row plus learned position row; franken_ocr decoder_qwen2.rs: token row only).
// A token of -1 in the step description means the slot's previous greedy pick.
__global__ void k_embed(const float* __restrict__ E, const float* __restrict__ P, const StepMeta* meta,
                        const int* __restrict__ last_tok, float* __restrict__ x, int d, int* __restrict__ table) {
    pdl_wait();
    // page-table entries of pages this step starts (a paged cache), before any kernel of the
    // step reads them
    if (table && blockIdx.x == 0)
        for (int i = threadIdx.x; i < meta->n_upd; i += blockDim.x) table[meta->upd_idx[i]] = meta->upd_page[i];
    const int b = blockIdx.x;
    if (b >= meta->B) return;
    int tok = meta->tok[b];
    if (tok < 0) tok = last_tok[meta->slot[b]];
    const float4* e = reinterpret_cast<const float4*>(E + static_cast<long long>(tok) * d);
    const float4* p = P ? reinterpret_cast<const float4*>(P + static_cast<long long>(meta->pos[b]) * d) : nullptr;
    float4* o = reinterpret_cast<float4*>(x + static_cast<long long>(b) * d);
    for (int i = threadIdx.x; i < d / 4; i += blockDim.x) {
        float4 v = e[i];
        if (p) {
            const float4 q = p[i];
            v.x = __fadd_rn(v.x, q.x);
            v.y = __fadd_rn(v.y, q.y);
            v.z = __fadd_rn(v.z, q.z);
            v.w = __fadd_rn(v.w, q.w);
        }
        o[i] = v;
    }
    pdl_launch_dependents();
}

// Page-table entries of a step description, applied on their own (before a K/V row copy).
__global__ void k_table_update(const StepMeta* meta, int* __restrict__ table) {
    for (int i = threadIdx.x; i < meta->n_upd; i += blockDim.x) table[meta->upd_idx[i]] = meta->upd_page[i];
}

// Token-major rows [L, n, H*64] <-> the head-first cache (dense or paged), bit for bit.
// dir 0: rows -> cache (KV append / seed); dir 1: cache -> rows (read back).
// The step description's page-table updates are applied first (a paged cache).
__global__ void k_kv_copy(float* __restrict__ cache, float* __restrict__ rows, int dir, long long layer_stride,
                          KvMap m, int slot, int start, int n, int d, int layer0) {
    const int r = blockIdx.x;        // row within [0, n)
    const int l = blockIdx.y;        // layer offset
    const long long lay = layer0 + l;
    int page, pr;
    kv_page_of(m, slot, start + r, page, pr);
    float* base = cache + lay * layer_stride;
    float* rrow = rows + (static_cast<long long>(l) * n + r) * d;
    for (int e = threadIdx.x; e < d / 4; e += blockDim.x) {
        const int col = e * 4, h = col >> 6, i = col & 63;
        float4* c = reinterpret_cast<float4*>(base + kv_page_off(m, page, h, pr) + i);
        float4* t = reinterpret_cast<float4*>(rrow + col);
        if (dir == 0)
            *c = *t;
        else
            *t = *c;
    }
}

// Cross-attention K or V for one stream and layer: C = enc W^T + b (W f32, or int8 rows
// times a per-row scale), written head-first [H][enc_len][64] (cera whisper.rs,
// `precompute_cross_attention`). Plain 64 x 64 register-tiled SIMT GEMM; runs once per
// stream at prefill, outside the decode step.
template <typename WT>
__global__ void __launch_bounds__(256) k_cross_kv(const float* __restrict__ enc, const WT* __restrict__ W,
                                                  const float* __restrict__ scale, const float* __restrict__ bias,
                                                  float* __restrict__ out, int M, int N, int K) {
    __shared__ float sA[16][64 + 4];
    __shared__ float sB[16][64 + 4];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += 16) {
        for (int e = threadIdx.x; e < 64 * 16; e += 256) {
            const int r = e >> 4, kk = e & 15;
            const int m = m0 + r, n = n0 + r, k = k0 + kk;
            sA[kk][r] = (m < M && k < K) ? enc[static_cast<long long>(m) * K + k] : 0.0f;
            sB[kk][r] = (n < N && k < K) ? static_cast<float>(W[static_cast<long long>(n) * K + k]) : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float av[4], bv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) av[i] = sA[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) bv[j] = sB[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n >= N) continue;
            float y = acc[i][j];
            if (scale) y *= scale[n];
            if (bias) y += bias[n];
            out[(static_cast<long long>(n >> 6) * M + m) * kHeadDim + (n & 63)] = y;
        }
    }
}

}  // namespace dec
