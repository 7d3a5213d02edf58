// Weight-streaming projection kernels for small batches: y[b, n] = sum_k x[b, k] W[n, k].
//
// Each warp owns two weight rows at a time (a "task") and streams them from HBM
// with 16-byte non-allocating loads, lane l covering bytes [16 l, 16 l + 16) of
// every 512-byte run of the row. The (normalised, optionally int8-quantised)
// activation rows of the batch tile sit in shared memory and are reused by every
// task of the CTA. Per-lane partial sums for the 2 x BT outputs of a task are
// reduced with a halving transpose, which leaves each output in one lane for the
// fused epilogue.
//
// Prologues (per activation row, computed by every CTA from the raw residual
// stream so that no separate norm kernel runs):
//   PRO_NONE  x as is
//   PRO_LN    LayerNorm (x - mean) / sqrt(var + eps) * g + b  (cera whisper.rs, layer_norm_inplace)
//   PRO_RMS   RMSNorm x / sqrt(mean(x^2) + eps) * w             (franken_ocr decoder_qwen2.rs, family_norm)
//   ACT_I8    then per-row symmetric int8 quantisation with ties to even:
//             inv = 127 / amax, q = rint(x * inv), a = amax / 127  (decoder_qwen2.rs, quantize_row_i8_te)
// Weight formats: f32; int8 with per-row scale and f32 activations (W8A32,
// lattice-inference cpu_q8.rs matmul_bt_q8); int8 with int8 activations and int32
// dp4a accumulation (W8A8, decoder_qwen2.rs gemv_i8_bias_prequant), dequantised as
// float(acc) * (a * s_n) + bias_n.
// Epilogues: store, residual add, GELU(tanh), Q/K/V split with NEOX RoPE and KV
// scatter, SwiGLU (silu(gate) * up), LM head logits with a fused greedy argmax.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace dec {

enum Pro { PRO_NONE = 0, PRO_LN = 1, PRO_RMS = 2, PRO_RAW_I8 = 3 };
enum Epi { EPI_STORE = 0, EPI_RESID = 1, EPI_GELU = 2, EPI_QKV = 3, EPI_SWIGLU = 4, EPI_HEAD = 5, EPI_I32 = 6 };
enum RowMap { MAP_ADJ = 0, MAP_ROPE = 1, MAP_DUAL = 2 };

constexpr int kGemvWarps = 4;
constexpr int kGemvThreads = kGemvWarps * 32;

struct GemvArgs {
    const float* x;          // activation rows (f32), row b at x + b * x_ld
    const int8_t* xq;        // PRO_RAW_I8: int8 activation rows
    int x_ld;
    const float* norm_w;
    const float* norm_b;
    float eps;
    int K, N;
    int B;                   // rows in the whole batch
    const void* W;           // [N, K] row-major
    const void* W2;          // MAP_DUAL second matrix (SwiGLU up)
    const float* scale;      // per-row scales (int8 weights)
    const float* scale2;
    const float* bias;
    float* out;              // STORE/GELU/SWIGLU/QKV(q)/HEAD(logits, may be null)/RESID(target)
    int out_ld;
    int* out_i32;            // EPI_I32
    // EPI_QKV
    float* kc;               // this layer's self K cache base
    float* vc;
    long long slot_stride;
    int ld;                  // cache rows per (slot, head)
    int d;                   // model width (q/k/v section size)
    const float2* rope;      // [pos][32] (cos, sin), null = no RoPE
    // EPI_HEAD
    unsigned long long* keys;  // [B] packed argmax keys, zero between launches
    int* counter;              // CTA arrival count, zero between launches
    int* argmax_out;           // [B] or null
    int* last_tok;             // [slots]
    const StepMeta* meta;
};

template <typename WT>
struct WVec;
template <>
struct WVec<float> {
    static constexpr int kElems = 4;
};
template <>
struct WVec<int8_t> {
    static constexpr int kElems = 16;
};

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ float norm_value(int pro, float x, float mu, float rstd, const float* g,
                                            const float* beta, int k) {
    if (pro == PRO_LN) {
        return __fadd_rn(__fmul_rn(__fmul_rn(__fsub_rn(x, mu), rstd), g[k]), beta[k]);
    } else if (pro == PRO_RMS) {
        return __fmul_rn(__fmul_rn(x, rstd), g[k]);
    }
    return x;
}

__device__ __forceinline__ int quant_i8(float y, float inv) {
    const float r = rintf(__fmul_rn(y, inv));
    return static_cast<int>(fminf(fmaxf(r, -127.0f), 127.0f));
}

// dot of 16 bytes of weights against activation elements [k, k + elems)
template <typename WT, bool I8>
struct Dot;

template <>
struct Dot<float, false> {
    __device__ __forceinline__ static void run(const uint4& w, const float* xs, float& acc) {
        const float4 xv = *reinterpret_cast<const float4*>(xs);
        acc = fmaf(__uint_as_float(w.x), xv.x, acc);
        acc = fmaf(__uint_as_float(w.y), xv.y, acc);
        acc = fmaf(__uint_as_float(w.z), xv.z, acc);
        acc = fmaf(__uint_as_float(w.w), xv.w, acc);
    }
};

__device__ __forceinline__ void acc_i8x4_f32(uint32_t w, const float4& xv, float& acc) {
    acc = fmaf(static_cast<float>(static_cast<int>(w << 24) >> 24), xv.x, acc);
    acc = fmaf(static_cast<float>(static_cast<int>(w << 16) >> 24), xv.y, acc);
    acc = fmaf(static_cast<float>(static_cast<int>(w << 8) >> 24), xv.z, acc);
    acc = fmaf(static_cast<float>(static_cast<int>(w) >> 24), xv.w, acc);
}

template <>
struct Dot<int8_t, false> {
    __device__ __forceinline__ static void run(const uint4& w, const float* xs, float& acc) {
        const float4* x4 = reinterpret_cast<const float4*>(xs);
        acc_i8x4_f32(w.x, x4[0], acc);
        acc_i8x4_f32(w.y, x4[1], acc);
        acc_i8x4_f32(w.z, x4[2], acc);
        acc_i8x4_f32(w.w, x4[3], acc);
    }
};

template <>
struct Dot<int8_t, true> {
    __device__ __forceinline__ static void run(const uint4& w, const int8_t* xs, int& acc) {
        const int4 xv = *reinterpret_cast<const int4*>(xs);
        acc = __dp4a(static_cast<int>(w.x), xv.x, acc);
        acc = __dp4a(static_cast<int>(w.y), xv.y, acc);
        acc = __dp4a(static_cast<int>(w.z), xv.z, acc);
        acc = __dp4a(static_cast<int>(w.w), xv.w, acc);
    }
};

// Shared-memory bytes of the activation tile for a K chunk.
template <int BT, bool I8>
__host__ __device__ constexpr size_t gemv_xtile_bytes(int kc) {
    return static_cast<size_t>(BT) * kc * (I8 ? 1 : 4);
}

template <int BT, typename WT, bool I8, int PRO, int EPI, int MAP>
__global__ void __launch_bounds__(kGemvThreads) k_gemv(const GemvArgs a, int KC) {
    using AccT = typename std::conditional<I8, int, float>::type;
    using XT = typename std::conditional<I8, int8_t, float>::type;
    constexpr int VE = WVec<WT>::kElems;
    constexpr int NV = 2 * BT;                 // outputs per task
    constexpr int NC = NV > 32 ? NV / 32 : 1;  // 32-value chunks
    constexpr int NVC = NV > 32 ? 32 : NV;
    constexpr int SH = transpose_shift<NVC>();
    static_assert(!(I8 && !std::is_same<WT, int8_t>::value), "int8 activations need int8 weights");

    extern __shared__ __align__(16) unsigned char gemv_smem[];
    XT* sX = reinterpret_cast<XT*>(gemv_smem);
    __shared__ float s_mu[BT], s_rstd[BT], s_inv[BT], s_a[BT];
    __shared__ unsigned long long s_key[BT];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b0 = blockIdx.y * BT;        // first batch row of this CTA's batch tile
    const int nb = min(BT, a.B - b0);  // live rows of this batch tile
    const int n_tasks = (MAP == MAP_DUAL) ? a.N : (a.N + 1) / 2;
    const int nchunks = (a.K + KC - 1) / KC;

    pdl_wait();

    // ---- per-row statistics over the full K ----
    if (PRO != PRO_RAW_I8) {
        for (int b = warp; b < BT; b += kGemvWarps) {
            float mu = 0.0f, rstd = 1.0f, inv = 0.0f, ascale = 0.0f;
            if (b < nb) {
                const float* xr = a.x + static_cast<long long>(b0 + b) * a.x_ld;
                if (PRO == PRO_LN) {
                    float sum = 0.0f;
                    for (int k = lane; k < a.K; k += 32) sum += xr[k];
                    sum = warp_sum(sum);
                    mu = sum / static_cast<float>(a.K);
                    float var = 0.0f;
                    for (int k = lane; k < a.K; k += 32) {
                        const float dv = xr[k] - mu;
                        var = fmaf(dv, dv, var);
                    }
                    var = warp_sum(var) / static_cast<float>(a.K);
                    rstd = 1.0f / sqrtf(var + a.eps);
                } else if (PRO == PRO_RMS) {
                    float ss = 0.0f;
                    for (int k = lane; k < a.K; k += 32) ss = fmaf(xr[k], xr[k], ss);
                    ss = warp_sum(ss) / static_cast<float>(a.K);
                    rstd = 1.0f / sqrtf(ss + a.eps);
                }
                if (I8) {
                    float amax = 0.0f;
                    for (int k = lane; k < a.K; k += 32)
                        amax = fmaxf(amax, fabsf(norm_value(PRO, xr[k], mu, rstd, a.norm_w, a.norm_b, k)));
                    amax = warp_max(amax);
                    inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
                    ascale = __fdiv_rn(amax, 127.0f);
                }
            }
            if (lane == 0) {
                s_mu[b] = mu;
                s_rstd[b] = rstd;
                s_inv[b] = inv;
                s_a[b] = ascale;
            }
        }
    }
    if (EPI == EPI_HEAD && tid < BT) s_key[tid] = 0ull;
    __syncthreads();

    auto stage_chunk = [&](int k0, int kc) {
        // activation tile [BT][kc] for columns [k0, k0 + kc); rows >= nb are zero
        const int total = BT * kc;
        for (int e = tid; e < total; e += kGemvThreads) {
            const int b = e / kc, kk = e - b * kc, k = k0 + kk;
            if (PRO == PRO_RAW_I8) {
                sX[e] = (b < nb) ? static_cast<XT>(a.xq[static_cast<long long>(b0 + b) * a.x_ld + k]) : XT(0);
            } else {
                float y = 0.0f;
                if (b < nb)
                    y = norm_value(PRO, a.x[static_cast<long long>(b0 + b) * a.x_ld + k], s_mu[b], s_rstd[b],
                                   a.norm_w, a.norm_b, k);
                if (I8)
                    sX[e] = static_cast<XT>(b < nb ? quant_i8(y, s_inv[b]) : 0);
                else
                    sX[e] = static_cast<XT>(y);
            }
        }
    };

    // per-lane running argmax keys for the head epilogue
    unsigned long long best[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) best[c] = 0ull;

    auto rows_of = [&](int task, int& r0, int& r1) {
        if (MAP == MAP_ROPE) {
            const int hb = task >> 5, i = task & 31;
            r0 = hb * 64 + i;
            r1 = r0 + 32;
        } else if (MAP == MAP_DUAL) {
            r0 = task;
            r1 = task;
        } else {
            r0 = 2 * task;
            r1 = 2 * task + 1;
        }
    };

    auto accumulate = [&](int r0, int r1, int k0, int kc, AccT (&acc)[2][BT]) {
        const WT* W0 = reinterpret_cast<const WT*>(a.W) + static_cast<long long>(r0) * a.K + k0;
        const WT* W1 = reinterpret_cast<const WT*>(MAP == MAP_DUAL ? a.W2 : a.W) +
                       static_cast<long long>(r1) * a.K + k0;
        const bool has1 = r1 < a.N;
        constexpr int U = 4;
        for (int kk = lane * VE; kk < kc; kk += 32 * VE * U) {
            uint4 w0[U], w1[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int k = kk + u * 32 * VE;
                if (k < kc) {
                    w0[u] = ldg_stream(W0 + k);
                    w1[u] = has1 ? ldg_stream(W1 + k) : make_uint4(0, 0, 0, 0);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int k = kk + u * 32 * VE;
                if (k < kc) {
#pragma unroll
                    for (int b = 0; b < BT; ++b) {
                        const XT* xs = sX + b * kc + k;
                        Dot<WT, I8>::run(w0[u], xs, acc[0][b]);
                        Dot<WT, I8>::run(w1[u], xs, acc[1][b]);
                    }
                }
            }
        }
    };

    auto epilogue = [&](int task, int r0, int r1, AccT (&acc)[2][BT]) {
        // flatten value index v = r + 2 b and reduce across the warp
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            AccT vals[NVC];
#pragma unroll
            for (int j = 0; j < NVC; ++j) {
                const int v = c * 32 + j;
                vals[j] = acc[v & 1][v >> 1];
            }
            const AccT red = warp_reduce_transpose<NVC>(vals);
            const int v = c * 32 + (lane >> SH);
            const int r = v & 1, b = v >> 1;
            const bool primary = (lane & ((1 << SH) - 1)) == 0;
            const int n = r ? r1 : r0;
            const bool live = (b < nb) && (n < a.N);
            // dequantise
            float y;
            if (EPI == EPI_I32) {
                y = 0.0f;  // raw accumulators only: no scales exist for this epilogue
            } else if (I8) {
                const float* sc = (MAP == MAP_DUAL && r) ? a.scale2 : a.scale;
                y = __fmul_rn(static_cast<float>(red), __fmul_rn(s_a[b], sc[live ? n : 0]));
            } else {
                y = static_cast<float>(red);
                if (std::is_same<WT, int8_t>::value) y = __fmul_rn(y, a.scale[live ? n : 0]);
            }
            if (EPI != EPI_HEAD && EPI != EPI_SWIGLU && EPI != EPI_I32 && a.bias != nullptr && live)
                y = __fadd_rn(y, a.bias[n]);
            // partner value (other row of the pair, same batch row)
            const float yp = __shfl_xor_sync(0xffffffffu, y, 1 << SH);
            const int gb = b0 + b;
            if (EPI == EPI_I32) {
                if (primary && live) a.out_i32[static_cast<long long>(gb) * a.out_ld + n] = static_cast<int>(red);
            } else if (EPI == EPI_STORE) {
                if (primary && live) a.out[static_cast<long long>(gb) * a.out_ld + n] = y;
            } else if (EPI == EPI_RESID) {
                if (primary && live) {
                    float* p = a.out + static_cast<long long>(gb) * a.out_ld + n;
                    *p = __fadd_rn(*p, y);
                }
            } else if (EPI == EPI_GELU) {
                if (primary && live) a.out[static_cast<long long>(gb) * a.out_ld + n] = gelu_tanh_f(y);
            } else if (EPI == EPI_SWIGLU) {
                // r = 0 holds gate row n, its partner holds up row n
                if (primary && live && r == 0)
                    a.out[static_cast<long long>(gb) * a.out_ld + n] = __fmul_rn(silu_f(y), yp);
            } else if (EPI == EPI_QKV) {
                const int sec = n / a.d, within = n - sec * a.d;
                const int hh = within >> 6, i = within & 63;
                float val = y;
                if (a.rope != nullptr && sec < 2) {
                    const float2 cs = a.rope[static_cast<long long>(a.meta->pos[gb < a.B ? gb : 0]) * 32 + (i & 31)];
                    // pair (i, i + 32): x_i' = x_i c - x_{i+32} s ; x_{i+32}' = x_i s + x_{i+32} c
                    if (i < 32)
                        val = __fsub_rn(__fmul_rn(y, cs.x), __fmul_rn(yp, cs.y));
                    else
                        val = __fadd_rn(__fmul_rn(yp, cs.y), __fmul_rn(y, cs.x));
                }
                if (primary && live) {
                    if (sec == 0) {
                        a.out[static_cast<long long>(gb) * a.out_ld + within] = val;
                    } else {
                        const int slot = a.meta->slot[gb], row = a.meta->len[gb];
                        float* cache = (sec == 1) ? a.kc : a.vc;
                        cache[slot * a.slot_stride + (static_cast<long long>(hh) * a.ld + row) * kHeadDim + i] = val;
                    }
                }
            } else if (EPI == EPI_HEAD) {
                if (primary && live && a.out != nullptr) a.out[static_cast<long long>(gb) * a.out_ld + n] = y;
                if (live) {
                    const unsigned long long key = argmax_key(y, n);
                    best[c] = key > best[c] ? key : best[c];
                }
            }
        }
    };

    if (nchunks == 1) {
        stage_chunk(0, a.K);
        __syncthreads();
        for (int task = blockIdx.x * kGemvWarps + warp; task < n_tasks; task += gridDim.x * kGemvWarps) {
            int r0, r1;
            rows_of(task, r0, r1);
            AccT acc[2][BT];
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int b = 0; b < BT; ++b) acc[r][b] = AccT(0);
            accumulate(r0, r1, 0, a.K, acc);
            epilogue(task, r0, r1, acc);
        }
    } else {
        // one task per warp; the activation tile is staged chunk by chunk
        const int task = blockIdx.x * kGemvWarps + warp;
        int r0 = 0, r1 = 0;
        const bool has_task = task < n_tasks;
        if (has_task) rows_of(task, r0, r1);
        AccT acc[2][BT];
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int b = 0; b < BT; ++b) acc[r][b] = AccT(0);
        for (int c = 0; c < nchunks; ++c) {
            const int k0 = c * KC, kc = min(KC, a.K - k0);
            __syncthreads();
            stage_chunk(k0, kc);
            __syncthreads();
            if (has_task) {
                accumulate(r0, r1, k0, kc, acc);
            }
        }
        if (has_task) epilogue(task, r0, r1, acc);
    }
    pdl_launch_dependents();

    if (EPI == EPI_HEAD) {
        // fold the two rows of each batch row, then the CTA, then the grid
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            unsigned long long o = __shfl_xor_sync(0xffffffffu, best[c], 1 << SH);
            best[c] = o > best[c] ? o : best[c];
            const int v = c * 32 + (lane >> SH);
            const int b = v >> 1;
            if ((lane & ((1 << SH) - 1)) == 0 && (v & 1) == 0 && b < nb && best[c] != 0ull)
                atomicMax(&s_key[b], best[c]);
        }
        __syncthreads();
        if (tid < nb && s_key[tid] != 0ull) atomicMax(&a.keys[b0 + tid], s_key[tid]);
        __shared__ int s_last;
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            const int total = gridDim.x * gridDim.y;
            s_last = (atomicAdd(a.counter, 1) == total - 1);
        }
        __syncthreads();
        if (s_last) {
            __threadfence();
            for (int b = tid; b < a.B; b += kGemvThreads) {
                const unsigned long long k = atomicExch(&a.keys[b], 0ull);
                const int idx = (k == 0ull) ? 0 : argmax_key_index(k);
                if (a.argmax_out) a.argmax_out[b] = idx;
                if (a.last_tok) a.last_tok[a.meta->slot[b]] = idx;
            }
            if (tid == 0) *a.counter = 0;
        }
    }
}

}  // namespace dec
