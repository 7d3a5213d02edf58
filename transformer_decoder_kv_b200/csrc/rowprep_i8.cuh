// Per-row int8 activation quantisation for the W8A8 tensor-core projections: one warp per
// row (optionally after RMSNorm or LayerNorm), inv = 127 / amax, q = rint(x * inv) with ties
// to even, a = amax / 127 (franken_ocr decoder_qwen2.rs, quantize_row_i8_te), with the
// CUDA-core projection prologue's arithmetic and reduction order, so that both paths
// produce the same codes and scales.
#pragma once

#include "common.cuh"
#include "gemv.cuh"

namespace dec {

// Per-row int8 quantisation (optionally after RMSNorm or LayerNorm), one warp per row,
// with the arithmetic and reduction order of the CUDA-core kernel's prologue so that both
// paths produce the same codes and scales.
// Rows of up to kRowprepRegK4 float4 per lane stay in registers: the row is read from global
// memory once instead of once per pass; every pass visits the elements in the same order
// (element lane + 32 j, j ascending) whether they come from registers or from memory.
constexpr int kRowprepRegK4 = 24;   // K <= 32 * 24 * 4 = 3072

template <int PRO, class Get>
__device__ __forceinline__ float rowprep_i8_passes(Get get, int K4, int K, int lane, const float4* g4,
                                                   const float4* be4, float eps, uint32_t* q, int jmax) {
    float mu = 0.0f, rstd = 1.0f;
    if (PRO == PRO_LN) {
        float sum = 0.0f;
        for (int j = 0; j < jmax; ++j)
            if (lane + 32 * j < K4) {
                const float4 v = get(j);
                sum += (v.x + v.y) + (v.z + v.w);
            }
        mu = warp_sum(sum) / static_cast<float>(K);
        float var = 0.0f;
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
        const int k = lane + 32 * j;
        const float4 v = get(j);
        float4 g = make_float4(1.f, 1.f, 1.f, 1.f), be = make_float4(0.f, 0.f, 0.f, 0.f);
        if (PRO != PRO_NONE) g = g4[k];
        if (PRO == PRO_LN) be = be4[k];
        return make_float4(norm_value(PRO, v.x, mu, rstd, g.x, be.x), norm_value(PRO, v.y, mu, rstd, g.y, be.y),
                           norm_value(PRO, v.z, mu, rstd, g.z, be.z), norm_value(PRO, v.w, mu, rstd, g.w, be.w));
    };
    float amax = 0.0f;
    for (int j = 0; j < jmax; ++j)
        if (lane + 32 * j < K4) {
            const float4 y = normed(j);
            amax = fmaxf(amax, fabsf(y.x));
            amax = fmaxf(amax, fabsf(y.y));
            amax = fmaxf(amax, fabsf(y.z));
            amax = fmaxf(amax, fabsf(y.w));
        }
    amax = warp_max(amax);
    const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
    for (int j = 0; j < jmax; ++j)
        if (lane + 32 * j < K4) {
            const float4 y = normed(j);
            q[lane + 32 * j] = (static_cast<uint32_t>(quant_i8(y.x, inv)) & 0xffu) |
                               ((static_cast<uint32_t>(quant_i8(y.y, inv)) & 0xffu) << 8) |
                               ((static_cast<uint32_t>(quant_i8(y.z, inv)) & 0xffu) << 16) |
                               ((static_cast<uint32_t>(quant_i8(y.w, inv)) & 0xffu) << 24);
        }
    return amax;
}

template <int PRO>
__global__ void __launch_bounds__(128) k_rowprep_i8(const float* __restrict__ x, int x_ld,
                                                    const float* __restrict__ gw, const float* __restrict__ gb,
                                                    float eps, int K, int B, int8_t* __restrict__ xq,
                                                    float* __restrict__ xs) {
    // the norm's weight (and LayerNorm bias) rows do not depend on the previous kernel: they
    // are copied into shared memory before the dependency wait
    extern __shared__ float4 rp_norm[];
    const int K4 = K >> 2;
    if (PRO != PRO_NONE)
        for (int i = threadIdx.x; i < K4; i += blockDim.x) {
            rp_norm[i] = reinterpret_cast<const float4*>(gw)[i];
            if (PRO == PRO_LN) rp_norm[K4 + i] = reinterpret_cast<const float4*>(gb)[i];
        }
    pdl_launch_dependents();
    pdl_wait();
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.x * 4 + (threadIdx.x >> 5);
    if (b >= B) return;
    const float4* xr = reinterpret_cast<const float4*>(x + static_cast<long long>(b) * x_ld);
    const float4* g4 = rp_norm;
    const float4* be4 = rp_norm + K4;
    uint32_t* q = reinterpret_cast<uint32_t*>(xq + static_cast<long long>(b) * K);
    float amax;
    if (K4 <= 32 * kRowprepRegK4) {
        float4 rv[kRowprepRegK4];
#pragma unroll
        for (int j = 0; j < kRowprepRegK4; ++j)
            rv[j] = lane + 32 * j < K4 ? xr[lane + 32 * j] : make_float4(0.f, 0.f, 0.f, 0.f);
        // every loop below is fully unrolled over the compile-time bound, so rv stays in registers
        amax = rowprep_i8_passes<PRO>([&](int j) { return rv[j]; }, K4, K, lane, g4, be4, eps, q, kRowprepRegK4);
    } else {
        amax = rowprep_i8_passes<PRO>([&](int j) { return xr[lane + 32 * j]; }, K4, K, lane, g4, be4, eps, q,
                                      (K4 + 31) / 32);
    }
    if (lane == 0) xs[b] = __fdiv_rn(amax, 127.0f);
}

template <int PRO>
cudaError_t rowprep_i8_launch(const GemvArgs& g, int8_t* xq, float* xs, cudaStream_t st);

#ifdef DEC_ROWPREP_I8_DEFINE

template <int PRO>
cudaError_t rowprep_i8_launch(const GemvArgs& g, int8_t* xq, float* xs, cudaStream_t st) {
    if (g.K % 16 != 0 || size_t(g.K) * 8 > size_t(227 * 1024)) return cudaErrorNotSupported;
    thread_local int attr_dev = -1;
    const cudaError_t e = prefer_max_shared_once(k_rowprep_i8<PRO>, attr_dev, 227 * 1024);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((g.B + 3) / 4);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = size_t(g.K) * 4 * (PRO == PRO_LN ? 2 : (PRO == PRO_RMS ? 1 : 0));
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_rowprep_i8<PRO>, g.x, g.x_ld, g.norm_w, g.norm_b, g.eps, g.K, g.B, xq, xs);
}

#define DEC_ROWPREP_I8_INSTANTIATE(PRO) \
    template cudaError_t rowprep_i8_launch<PRO>(const GemvArgs&, int8_t*, float*, cudaStream_t);

#endif  // DEC_ROWPREP_I8_DEFINE

}  // namespace dec
