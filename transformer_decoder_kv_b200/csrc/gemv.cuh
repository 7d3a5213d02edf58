// Weight-streaming projection kernels for small batches: y[b, n] = sum_k x[b, k] W[n, k].
//
// Work unit: a block of 4 tasks = 8 weight rows (each warp owns one task = two
// rows). CTAs are persistent over blocks. The rows of a block are moved from HBM
// into a shared-memory ring by one thread with 1-D bulk async copies (one per row
// and K chunk) completing on an mbarrier per stage; weights do not depend on the
// previous kernel, so the first stages are issued before the programmatic-
// dependent-launch wait and overlap the previous kernel's tail. The
// (normalised, optionally int8-quantised) activation rows of the batch tile are
// staged once per CTA after the wait, with 16-byte loads, and reused by every
// block. Per-lane partial sums for the 2 x BT outputs of a task are reduced with a
// halving transpose, which leaves each output in one lane for the fused epilogue.
//
// Prologues (per activation row, computed by every CTA from the raw residual
// stream so that no separate norm kernel runs):
//   PRO_NONE  x as is
//   PRO_LN    LayerNorm (x - mean) / sqrt(var + eps) * g + b  (cera whisper.rs, layer_norm_inplace)
//   PRO_RMS   RMSNorm x / sqrt(mean(x^2) + eps) * w             (franken_ocr decoder_qwen2.rs, family_norm)
//   I8        then per-row symmetric int8 quantisation with ties to even:
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
constexpr int kGemvRowsPerBlock = 2 * kGemvWarps;
constexpr int kGemvMaxStages = 8;
constexpr int kGemvStageBytes = 16 * 1024;   // weight bytes per stage at most

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
    KvMap kv;                // where each (slot, head, row) of the cache lives
    int d;                   // model width (the q section's size)
    int kvd;                 // K and V section size (kv heads x 64; d without grouped heads)
    const float2* rope;      // [pos][32] (cos, sin), null = no RoPE
    // EPI_HEAD
    unsigned long long* keys;  // [B] packed argmax keys, zero between launches
    int* counter;              // CTA arrival count, zero between launches
    int* argmax_out;           // [B] or null
    int* last_tok;             // [slots]
    const StepMeta* meta;
    int* err;                  // device status word
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

__device__ __forceinline__ float norm_value(int pro, float x, float mu, float rstd, float g, float beta) {
    if (pro == PRO_LN) return __fadd_rn(__fmul_rn(__fmul_rn(__fsub_rn(x, mu), rstd), g), beta);
    if (pro == PRO_RMS) return __fmul_rn(__fmul_rn(x, rstd), g);
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

// Warp roles: gemv_consumer_warps(BT) warps compute, one more warp moves weights.
// Batch tiles of 1-2 use 4 consumer warps and 8-row blocks, so that even a 1 MB
// matrix spreads over every SM; larger tiles use 8 consumer warps.
__host__ __device__ constexpr int gemv_consumer_warps(int bt) { return bt <= 2 ? 4 : 8; }
__host__ __device__ constexpr int gemv_threads(int bt) { return (gemv_consumer_warps(bt) + 1) * 32; }
// Rows per consumer-warp task: four for batch tiles 4 and 8 (more independent rows
// per warp), two otherwise (for 16 and 32 the R x BT accumulators bound the registers).
__host__ __device__ constexpr int gemv_rows_per_task(int bt) { return (bt == 4 || bt == 8) ? 4 : 2; }
// Weight bytes per pipeline stage at most.
__host__ __device__ constexpr int gemv_stage_bytes(int bt) { return bt <= 8 ? 32 * 1024 : 16 * 1024; }

// Pair p of a row map (MAP_ADJ: 2p, 2p+1; MAP_ROPE: the NEOX pair (i, i + 32) of one
// head; MAP_DUAL: row p of W and of W2). A task of R rows holds pairs R/2 t .. R/2 t + R/2 - 1.
template <int MAP>
__device__ __forceinline__ void pair_rows(int p, int& r0, int& r1) {
    if (MAP == MAP_ROPE) {
        const int hb = p >> 5, i = p & 31;
        r0 = hb * 64 + i;
        r1 = r0 + 32;
    } else if (MAP == MAP_DUAL) {
        r0 = p;
        r1 = p;
    } else {
        r0 = 2 * p;
        r1 = 2 * p + 1;
    }
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <int BT, typename WT, bool I8, int PRO, int EPI, int MAP>
__global__ void __launch_bounds__(gemv_threads(BT), 2) k_gemv(const GemvArgs a, int KC, int NS) {
    using AccT = typename std::conditional<I8, int, float>::type;
    using XT = typename std::conditional<I8, int8_t, float>::type;
    constexpr int NWC = gemv_consumer_warps(BT);
    constexpr int NT = gemv_threads(BT);
    constexpr int R = gemv_rows_per_task(BT);   // weight rows per warp task
    constexpr int P = R / 2;                    // row pairs per task
    constexpr int ROWS_PER_BLOCK = R * NWC;
    constexpr int VE = WVec<WT>::kElems;
    constexpr int NV = R * BT;                  // outputs per task
    constexpr int NC = NV > 32 ? NV / 32 : 1;   // 32-value chunks
    constexpr int NVC = NV > 32 ? 32 : NV;
    constexpr int SH = transpose_shift<NVC>();
    constexpr bool RAW_STAGE = I8 && PRO != PRO_RAW_I8;   // f32 rows staged apart from the int8 tile
    static_assert(!(I8 && !std::is_same<WT, int8_t>::value), "int8 activations need int8 weights");

    extern __shared__ __align__(128) unsigned char gemv_smem[];
    const int stage_bytes = ROWS_PER_BLOCK * KC * static_cast<int>(sizeof(WT));
    unsigned char* ring = gemv_smem;
    XT* sX = reinterpret_cast<XT*>(gemv_smem + static_cast<size_t>(NS) * stage_bytes);
    float* sXraw = RAW_STAGE ? reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(sX) +
                                                         static_cast<size_t>(BT) * a.K * sizeof(XT))
                             : reinterpret_cast<float*>(sX);
    // the norm's weight (and LayerNorm bias) rows, copied in before the dependency wait
    constexpr bool NORM_W = PRO == PRO_RMS || PRO == PRO_LN;
    float* sNw = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(sX) +
                                          static_cast<size_t>(BT) * a.K * sizeof(XT) +
                                          (RAW_STAGE ? static_cast<size_t>(BT) * a.K * 4 : 0));
    float* sNb = sNw + a.K;
    __shared__ __align__(8) uint64_t full[kGemvMaxStages];
    __shared__ __align__(8) uint64_t empty[kGemvMaxStages];
    __shared__ __align__(8) uint64_t bar_x, bar_g;
    __shared__ float s_mu[BT], s_rstd[BT], s_inv[BT], s_a[BT];
    __shared__ unsigned long long s_key[BT];
    __shared__ int s_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool producer = warp == NWC;
    const int b0 = blockIdx.y * BT;        // first batch row of this CTA's batch tile
    const int nb = min(BT, a.B - b0);      // live rows of this batch tile
    const int n_pairs = (MAP == MAP_DUAL) ? a.N : (a.N + 1) / 2;
    const int n_tasks = (n_pairs + P - 1) / P;
    const int n_blocks = (n_tasks + NWC - 1) / NWC;
    const int nkc = (a.K + KC - 1) / KC;
    const int my_blocks = blockIdx.x < n_blocks ? (n_blocks - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int n_items = my_blocks * nkc;

    // rows of task t, in pair order (-1 = no row)
    auto task_rows = [&](int task, int (&rows)[R]) {
#pragma unroll
        for (int q = 0; q < P; ++q) {
            const int p = task * P + q;
            int r0 = -1, r1 = -1;
            if (task < n_tasks && p < n_pairs) pair_rows<MAP>(p, r0, r1);
            rows[2 * q] = (r0 >= 0 && r0 < a.N) ? r0 : -1;
            rows[2 * q + 1] = (r1 >= 0 && r1 < a.N) ? r1 : -1;
        }
    };

    // ---- weight pipeline: item `it` = (block, K chunk) -> stage it % NS ----
    auto issue = [&](int it) {
        const int jb = blockIdx.x + (it / nkc) * gridDim.x;
        const int c = it % nkc;
        const int k0 = c * KC, kc = min(KC, a.K - k0);
        const uint32_t row_bytes = static_cast<uint32_t>(kc) * sizeof(WT);
        const int stage = it % NS;
        unsigned char* dst = ring + static_cast<size_t>(stage) * stage_bytes;
        uint32_t total = 0;
        for (int w = 0; w < NWC; ++w) {
            int rows[R];
            task_rows(jb * NWC + w, rows);
#pragma unroll
            for (int r = 0; r < R; ++r)
                if (rows[r] >= 0) total += row_bytes;
        }
        mbar_arrive_expect_tx(&full[stage], total);
        // slots in order; runs of consecutive full rows of one matrix move as one copy
        int run_row = -1, run_len = 0, run_slot = 0;
        const void* run_base = nullptr;
        auto flush = [&]() {
            if (run_len > 0) {
                const WT* g = reinterpret_cast<const WT*>(run_base) + static_cast<long long>(run_row) * a.K + k0;
                bulk_g2s(dst + static_cast<size_t>(run_slot) * KC * sizeof(WT), g, row_bytes * run_len, &full[stage]);
            }
            run_len = 0;
        };
        for (int w = 0; w < NWC; ++w) {
            int rows[R];
            task_rows(jb * NWC + w, rows);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int slot = w * R + r;
                const void* base = (MAP == MAP_DUAL && (r & 1)) ? a.W2 : a.W;
                if (rows[r] < 0) {
                    flush();
                    continue;
                }
                if (run_len > 0 && nkc == 1 && base == run_base && rows[r] == run_row + run_len &&
                    slot == run_slot + run_len) {
                    ++run_len;
                } else {
                    flush();
                    run_row = rows[r];
                    run_base = base;
                    run_slot = slot;
                    run_len = 1;
                }
            }
        }
        flush();
    };

    // weights do not depend on the previous kernel: start streaming before the wait
    int n_issued = 0;
    if (producer && lane == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], NWC);
        }
        mbar_init(&bar_x, 1);
        mbar_init(&bar_g, 1);
        mbar_fence_init();
        if (NORM_W) {
            const uint32_t nbytes = static_cast<uint32_t>(a.K) * 4;
            mbar_arrive_expect_tx(&bar_g, PRO == PRO_LN ? 2 * nbytes : nbytes);
            bulk_g2s(sNw, a.norm_w, nbytes, &bar_g);
            if (PRO == PRO_LN) bulk_g2s(sNb, a.norm_b, nbytes, &bar_g);
        }
        for (; n_issued < NS && n_issued < n_items; ++n_issued) issue(n_issued);
    }
    pdl_launch_dependents();
    pdl_wait();

    // ---- activation rows (they come from the previous kernel): one bulk copy per row ----
    const int in_elt = (PRO == PRO_RAW_I8) ? 1 : 4;
    if (producer && lane == 0) {
        const uint32_t row_bytes = static_cast<uint32_t>(a.K) * in_elt;
        mbar_arrive_expect_tx(&bar_x, row_bytes * nb);
        for (int b = 0; b < nb; ++b) {
            if (PRO == PRO_RAW_I8)
                bulk_g2s(reinterpret_cast<int8_t*>(sX) + static_cast<size_t>(b) * a.K,
                         a.xq + static_cast<long long>(b0 + b) * a.x_ld, row_bytes, &bar_x);
            else
                bulk_g2s(sXraw + static_cast<size_t>(b) * a.K, a.x + static_cast<long long>(b0 + b) * a.x_ld,
                         row_bytes, &bar_x);
        }
        s_flag = (mbar_wait_bounded(&bar_x, 0, a.err) && (!NORM_W || mbar_wait_bounded(&bar_g, 0, a.err))) ? 1 : 0;
    }
    __syncthreads();
    if (!s_flag) {
        if (producer && lane == 0) {
            for (int i2 = 0; i2 < n_issued; ++i2) mbar_wait_bounded(&full[i2], 0, nullptr);
            if (NORM_W) mbar_wait_bounded(&bar_g, 0, nullptr);
        }
        __syncthreads();
        return;
    }
    (void)mbar_try_wait(&bar_x, 0);
    if (NORM_W) (void)mbar_try_wait(&bar_g, 0);

    // ---- per-row statistics from shared memory ----
    // (the loops are unrolled so that several shared-memory loads are in flight; each lane
    // still accumulates its elements in the same order)
    if (PRO != PRO_RAW_I8 && !producer) {
        for (int b = warp; b < BT; b += NWC) {
            float mu = 0.0f, rstd = 1.0f, inv = 0.0f, ascale = 0.0f;
            if (b < nb) {
                const float4* xr = reinterpret_cast<const float4*>(sXraw + static_cast<size_t>(b) * a.K);
                const float4* g4 = reinterpret_cast<const float4*>(sNw);
                const float4* be4 = reinterpret_cast<const float4*>(sNb);
                const int K4 = a.K >> 2;
                if (PRO == PRO_LN) {
                    float sum = 0.0f;
#pragma unroll 4
                    for (int k = lane; k < K4; k += 32) {
                        const float4 v = xr[k];
                        sum += (v.x + v.y) + (v.z + v.w);
                    }
                    mu = warp_sum(sum) / static_cast<float>(a.K);
                    float var = 0.0f;
#pragma unroll 4
                    for (int k = lane; k < K4; k += 32) {
                        const float4 v = xr[k];
                        const float d0 = v.x - mu, d1 = v.y - mu, d2 = v.z - mu, d3 = v.w - mu;
                        var = fmaf(d0, d0, var);
                        var = fmaf(d1, d1, var);
                        var = fmaf(d2, d2, var);
                        var = fmaf(d3, d3, var);
                    }
                    var = warp_sum(var) / static_cast<float>(a.K);
                    rstd = 1.0f / sqrtf(var + a.eps);
                } else if (PRO == PRO_RMS) {
                    float ss = 0.0f;
#pragma unroll 4
                    for (int k = lane; k < K4; k += 32) {
                        const float4 v = xr[k];
                        ss = fmaf(v.x, v.x, ss);
                        ss = fmaf(v.y, v.y, ss);
                        ss = fmaf(v.z, v.z, ss);
                        ss = fmaf(v.w, v.w, ss);
                    }
                    ss = warp_sum(ss) / static_cast<float>(a.K);
                    rstd = 1.0f / sqrtf(ss + a.eps);
                }
                if (I8) {
                    float amax = 0.0f;
#pragma unroll 4
                    for (int k = lane; k < K4; k += 32) {
                        const float4 v = xr[k];
                        float4 g = make_float4(1.f, 1.f, 1.f, 1.f), be = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (PRO != PRO_NONE) g = g4[k];
                        if (PRO == PRO_LN) be = be4[k];
                        amax = fmaxf(amax, fabsf(norm_value(PRO, v.x, mu, rstd, g.x, be.x)));
                        amax = fmaxf(amax, fabsf(norm_value(PRO, v.y, mu, rstd, g.y, be.y)));
                        amax = fmaxf(amax, fabsf(norm_value(PRO, v.z, mu, rstd, g.z, be.z)));
                        amax = fmaxf(amax, fabsf(norm_value(PRO, v.w, mu, rstd, g.w, be.w)));
                    }
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

    // ---- normalise (and quantise) in shared memory; padding rows become zero ----
    if (PRO != PRO_RAW_I8 && (PRO != PRO_NONE || I8 || nb < BT)) {
        const int K4 = a.K >> 2;
        const int total = BT * K4;
        for (int e = tid; e < total; e += NT) {
            const int b = e / K4, k4 = e - b * K4;
            float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
            if (b < nb) {
                const float4 v = reinterpret_cast<const float4*>(sXraw)[e];
                float4 g = make_float4(1.f, 1.f, 1.f, 1.f), be = make_float4(0.f, 0.f, 0.f, 0.f);
                if (PRO != PRO_NONE) g = reinterpret_cast<const float4*>(sNw)[k4];
                if (PRO == PRO_LN) be = reinterpret_cast<const float4*>(sNb)[k4];
                y.x = norm_value(PRO, v.x, s_mu[b], s_rstd[b], g.x, be.x);
                y.y = norm_value(PRO, v.y, s_mu[b], s_rstd[b], g.y, be.y);
                y.z = norm_value(PRO, v.z, s_mu[b], s_rstd[b], g.z, be.z);
                y.w = norm_value(PRO, v.w, s_mu[b], s_rstd[b], g.w, be.w);
            }
            if (I8) {
                uint32_t pk = 0;
                if (b < nb) {
                    const float inv = s_inv[b];
                    pk = (static_cast<uint32_t>(quant_i8(y.x, inv)) & 0xffu) |
                         ((static_cast<uint32_t>(quant_i8(y.y, inv)) & 0xffu) << 8) |
                         ((static_cast<uint32_t>(quant_i8(y.z, inv)) & 0xffu) << 16) |
                         ((static_cast<uint32_t>(quant_i8(y.w, inv)) & 0xffu) << 24);
                }
                reinterpret_cast<uint32_t*>(sX)[e] = pk;
            } else {
                reinterpret_cast<float4*>(sX)[e] = y;
            }
        }
    } else if (PRO == PRO_RAW_I8 && nb < BT) {
        for (int e = nb * (a.K >> 2) + tid; e < BT * (a.K >> 2); e += NT)
            reinterpret_cast<uint32_t*>(sX)[e] = 0u;
    }
    __syncthreads();

    // per-lane running argmax keys for the head epilogue
    unsigned long long best[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) best[c] = 0ull;

    if (producer) {
        // refill each stage once all consumer warps have released it
        if (lane == 0) {
            for (int it = n_issued; it < n_items; ++it) {
                const int stage = it % NS;
                if (!mbar_wait_bounded(&empty[stage], static_cast<uint32_t>(it / NS - 1) & 1u, a.err)) break;
                issue(it);
                n_issued = it + 1;
            }
            // every copy issued has landed before the CTA may leave (bounded)
            for (int i2 = max(0, n_issued - NS); i2 < n_issued; ++i2)
                mbar_wait_bounded(&full[i2 % NS], static_cast<uint32_t>(i2 / NS) & 1u, nullptr);
        }
    } else {
        AccT acc[R][BT];
        struct EpiPre {
            float s, bias, prev;
            float2 cs;
            int page, row;
        } pre[NC];
        for (int it = 0; it < n_items; ++it) {
            const int stage = it % NS;
            const uint32_t phase = static_cast<uint32_t>(it / NS) & 1u;
            int ok = 1;
            if (lane == 0) ok = mbar_wait_bounded(&full[stage], phase, a.err) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (lane != 0) (void)mbar_try_wait(&full[stage], phase);
            const int jb = blockIdx.x + (it / nkc) * gridDim.x;
            const int c = it % nkc;
            const int k0 = c * KC, kc = min(KC, a.K - k0);
            const int task = jb * NWC + warp;
            if (c == 0) {
#pragma unroll
                for (int r = 0; r < R; ++r)
#pragma unroll
                    for (int b = 0; b < BT; ++b) acc[r][b] = AccT(0);
                // the epilogue's global inputs of this task (row scale, bias, residual value,
                // RoPE table entry, cache page) are loaded now, so that their latency hides
                // behind the dot products instead of following the reduction
                if (task < n_tasks) {
                    int rows[R];
                    task_rows(task, rows);
#pragma unroll
                    for (int cc = 0; cc < NC; ++cc) {
                        const int v = cc * 32 + (lane >> SH);
                        const int r = v % R, b = v / R;
                        const int n = rows[r];
                        const bool live = (b < nb) && (n >= 0);
                        const bool primary = (lane & ((1 << SH) - 1)) == 0;
                        const int gb = b0 + b;
                        const float* sc = (MAP == MAP_DUAL && (r & 1)) ? a.scale2 : a.scale;
                        pre[cc].s = (EPI != EPI_I32 && (I8 || std::is_same<WT, int8_t>::value)) ? sc[live ? n : 0]
                                                                                               : 1.0f;
                        pre[cc].bias = (EPI != EPI_HEAD && EPI != EPI_SWIGLU && EPI != EPI_I32 && a.bias != nullptr &&
                                        live)
                                           ? a.bias[n]
                                           : 0.0f;
                        pre[cc].prev = (EPI == EPI_RESID && primary && live)
                                           ? a.out[static_cast<long long>(gb) * a.out_ld + n]
                                           : 0.0f;
                        if (EPI == EPI_QKV) {
                            const int sec = n < a.d ? 0 : (n < a.d + a.kvd ? 1 : 2);
                            const int i = (n - (sec == 0 ? 0 : (sec == 1 ? a.d : a.d + a.kvd))) & 63;
                            pre[cc].cs = (a.rope != nullptr && sec < 2)
                                             ? a.rope[static_cast<long long>(a.meta->pos[gb < a.B ? gb : 0]) * 32 +
                                                      (i & 31)]
                                             : make_float2(1.0f, 0.0f);
                            pre[cc].page = 0;
                            pre[cc].row = 0;
                            if (primary && live && sec > 0)
                                kv_page_of(a.kv, a.meta->slot[gb], a.meta->len[gb], pre[cc].page, pre[cc].row);
                        }
                    }
                }
            }
            if (task < n_tasks) {
                const WT* wbase = reinterpret_cast<const WT*>(ring + static_cast<size_t>(stage) * stage_bytes) +
                                  static_cast<size_t>(R * warp) * KC;
                const XT* xbase = sX + k0;
#pragma unroll 2
                for (int kk = lane * VE; kk < kc; kk += 32 * VE) {
                    uint4 wv[R];
#pragma unroll
                    for (int r = 0; r < R; ++r)
                        wv[r] = *reinterpret_cast<const uint4*>(wbase + static_cast<size_t>(r) * KC + kk);
#pragma unroll
                    for (int b = 0; b < BT; ++b) {
                        const XT* xs = xbase + static_cast<size_t>(b) * a.K + kk;
#pragma unroll
                        for (int r = 0; r < R; ++r) Dot<WT, I8>::run(wv[r], xs, acc[r][b]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (task < n_tasks && c == nkc - 1) {
                int rows[R];
                task_rows(task, rows);
#pragma unroll
                for (int cc = 0; cc < NC; ++cc) {
                    AccT vals[NVC];
#pragma unroll
                    for (int j = 0; j < NVC; ++j) {
                        const int v = cc * 32 + j;
                        vals[j] = acc[v % R][v / R];
                    }
                    const AccT red = warp_reduce_transpose<NVC>(vals);
                    const int v = cc * 32 + (lane >> SH);
                    const int r = v % R, b = v / R;
                    const bool primary = (lane & ((1 << SH) - 1)) == 0;
                    const int n = rows[r];
                    const bool live = (b < nb) && (n >= 0);
                    float y;
                    if (EPI == EPI_I32) {
                        y = 0.0f;  // raw accumulators only: no scales exist for this epilogue
                    } else if (I8) {
                        y = __fmul_rn(static_cast<float>(red), __fmul_rn(s_a[b], pre[cc].s));
                    } else {
                        y = static_cast<float>(red);
                        if (std::is_same<WT, int8_t>::value) y = __fmul_rn(y, pre[cc].s);
                    }
                    if (EPI != EPI_HEAD && EPI != EPI_SWIGLU && EPI != EPI_I32 && a.bias != nullptr && live)
                        y = __fadd_rn(y, pre[cc].bias);
                    // partner value (other row of the pair, same batch row): value index v ^ 1
                    const float yp = __shfl_xor_sync(0xffffffffu, y, 1 << SH);
                    const int gb = b0 + b;
                    if (EPI == EPI_I32) {
                        if (primary && live)
                            a.out_i32[static_cast<long long>(gb) * a.out_ld + n] = static_cast<int>(red);
                    } else if (EPI == EPI_STORE) {
                        if (primary && live) a.out[static_cast<long long>(gb) * a.out_ld + n] = y;
                    } else if (EPI == EPI_RESID) {
                        if (primary && live) a.out[static_cast<long long>(gb) * a.out_ld + n] = __fadd_rn(pre[cc].prev, y);
                    } else if (EPI == EPI_GELU) {
                        if (primary && live) a.out[static_cast<long long>(gb) * a.out_ld + n] = gelu_tanh_f(y);
                    } else if (EPI == EPI_SWIGLU) {
                        // even r holds gate row n, its partner holds up row n
                        if (primary && live && (r & 1) == 0)
                            a.out[static_cast<long long>(gb) * a.out_ld + n] = __fmul_rn(silu_f(y), yp);
                    } else if (EPI == EPI_QKV) {
                        const int sec = n < a.d ? 0 : (n < a.d + a.kvd ? 1 : 2);
                        const int within = n - (sec == 0 ? 0 : (sec == 1 ? a.d : a.d + a.kvd));
                        const int hh = within >> 6, i = within & 63;
                        float val = y;
                        if (a.rope != nullptr && sec < 2) {
                            const float2 cs = pre[cc].cs;
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
                                float* cache = (sec == 1) ? a.kc : a.vc;
                                cache[kv_page_off(a.kv, pre[cc].page, hh, pre[cc].row) + i] = val;
                            }
                        }
                    } else if (EPI == EPI_HEAD) {
                        if (primary && live && a.out != nullptr)
                            a.out[static_cast<long long>(gb) * a.out_ld + n] = y;
                        if (live) {
                            const unsigned long long key = argmax_key(y, n);
                            best[cc] = key > best[cc] ? key : best[cc];
                        }
                    }
                }
            }
        }
    }

    if (EPI == EPI_HEAD) {
        // fold the rows of each batch row, then the CTA, then the grid
        __syncthreads();
        if (!producer) {
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                const int v = c * 32 + (lane >> SH);
                const int b = v / R;
                if ((lane & ((1 << SH) - 1)) == 0 && b < nb && best[c] != 0ull) atomicMax(&s_key[b], best[c]);
            }
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
            for (int b = tid; b < a.B; b += NT) {
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
