// Split-K decode attention over head-first K/V caches (self- and cross-attention).
//
// One query row per (stream b, head h) attends keys 0..n-1 of its own cache:
// s_j = (q . k_j) / 8, p = softmax(s) with the row max subtracted, out = sum_j p_j v_j
// (franken_ocr decoder_qwen2.rs, `decode_attn_head`; cera whisper.rs,
// `multi_head_attention`). A row whose softmax sum is not finite and positive
// gives zeros (lattice-inference cpu_q8.rs, full-attention step: fail closed).
//
// Work split: grid (S, H, B). CTA (s, h, b) takes a contiguous range of 64-key
// tiles of the (b, h) cache. Each tile of K and of V is one contiguous 16 KB run
// in the head-first layout, so one thread moves it into shared memory with a
// single bulk async copy completing on an mbarrier; three stages are in flight.
// Four warps share a tile, 16 keys each: lanes 0-15 / 16-31 take the low / high 32
// dims of one key, so a score needs one shuffle. Each warp keeps an online-softmax
// state (running max, sum, and two output dims per lane); warps merge through
// shared memory, and when a (b, h) row uses more than one CTA, partial states go
// to a scratch buffer and the last CTA to finish (an atomic arrival count, no
// waiting) merges them in split order and resets the count.
#pragma once

#include "common.cuh"

namespace dec {

constexpr int kAttnTile = 64;
constexpr int kAttnStages = 3;
constexpr int kAttnThreads = 128;
constexpr int kAttnPartStride = 68;  // m, l, 2 pad, o[64]
constexpr size_t kAttnSmemBytes = size_t(kAttnStages) * 2 * kAttnTile * kHeadDim * sizeof(float);

enum AttnMode { ATTN_SELF = 0, ATTN_CROSS = 1, ATTN_OP = 2 };

struct AttnArgs {
    const float* q;        // query of (b, h) at q + b * q_bstride + h * 64
    long long q_bstride;
    const float* k;        // this layer's cache base; (slot, h) block at slot * slot_stride + h * ld * 64
    const float* v;
    long long slot_stride;
    int ld;                // rows per (slot, head)
    int H;
    int mode;              // AttnMode
    int n_fixed;           // ATTN_CROSS: keys per row
    int batch;             // ATTN_OP: batch size
    const StepMeta* meta;  // ATTN_SELF / ATTN_CROSS
    const int* lens;       // ATTN_OP: keys per stream (device)
    float* out;            // output of (b, h) at out + b * out_bstride + h * 64
    long long out_bstride;
    float* part;           // [B * H * S * 68] partial states
    int* counters;         // [B * H] arrival counts, zero between launches
    int S;                 // splits (gridDim.x), the partial-state stride per row
    int tps;               // 64-key tiles per split; 0: ceil(tiles / S) per row
    int stages;            // shared-memory pipeline stages (1..3); 0: 3
    int* err;              // device status word
    int drop_first_copy;   // test hook: CTA (0, 0, 0) never issues its first tile's copies
    int kv_group;          // query heads per K/V head (grouped-query attention); 0 or 1: one each
    KvMap kv;              // ATTN_SELF with a paged cache: where each row lives (table null: dense)
};

// Rows [64 tile, 64 tile + 64) of one (slot, K/V head), clipped to n: one bulk copy each of K
// and V when the rows are contiguous (dense cache, Kb/Vb the head's first row), else one per
// page they span (paged cache, pages of 16, 32 or 64 rows).
// `drop`: announce the bytes but issue no copy, so that the tile's wait can only run out
// (the host-side fault injection of the failure-path tests; no memory is touched).
__device__ __forceinline__ void attn_issue(float* sK, float* sV, uint64_t* bar, const AttnArgs& a, const float* Kb,
                                           const float* Vb, int slot, int hk, int tile, int n, bool drop = false) {
    const int rows = min(kAttnTile, n - tile * kAttnTile);
    const uint32_t bytes = static_cast<uint32_t>(rows) * kHeadDim * sizeof(float);
    mbar_arrive_expect_tx(bar, 2 * bytes);
    if (drop) return;
    if (a.kv.table == nullptr) {
        bulk_g2s(sK, Kb + static_cast<long long>(tile) * kAttnTile * kHeadDim, bytes, bar);
        bulk_g2s(sV, Vb + static_cast<long long>(tile) * kAttnTile * kHeadDim, bytes, bar);
        return;
    }
    for (int r0 = 0; r0 < rows;) {
        int page, pr;
        kv_page_of(a.kv, slot, tile * kAttnTile + r0, page, pr);
        const int chunk = min(rows - r0, a.kv.page_rows - pr);
        const long long off = kv_page_off(a.kv, page, hk, pr);
        const uint32_t cb = static_cast<uint32_t>(chunk) * kHeadDim * sizeof(float);
        bulk_g2s(sK + r0 * kHeadDim, a.k + off, cb, bar);
        bulk_g2s(sV + r0 * kHeadDim, a.v + off, cb, bar);
        r0 += chunk;
    }
}

// Internal linkage: each translation unit that launches it carries its own copy.
static __global__ void __launch_bounds__(kAttnThreads) k_attention(const AttnArgs a) {
    extern __shared__ __align__(128) unsigned char attn_smem[];
    float* sK = reinterpret_cast<float*>(attn_smem);
    const int NS = (a.stages > 0 && a.stages <= kAttnStages) ? a.stages : kAttnStages;
    float* sV = sK + NS * kAttnTile * kHeadDim;
    __shared__ __align__(8) uint64_t bars[kAttnStages];
    __shared__ __align__(16) float sq[kHeadDim];
    __shared__ float wm[4], wl[4];
    __shared__ __align__(16) float wo[4][kHeadDim];
    __shared__ int s_flag;

    // The step description and cache rows older than this step were written before
    // the previous kernel ran; only the new row (self-attention) and q come from it.
    // Standalone calls wait first: their inputs may come from any kernel.
    if (a.mode == ATTN_OP) pdl_wait();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;

    int n, slot;
    if (a.mode == ATTN_OP) {
        if (b >= a.batch) return;
        n = min(max(a.lens[b], 0), a.ld);
        slot = b;
    } else {
        if (b >= a.meta->B) return;
        slot = a.meta->slot[b];
        n = (a.mode == ATTN_SELF) ? a.meta->len[b] + 1 : a.n_fixed;
    }
    float* outp = a.out + b * a.out_bstride + h * kHeadDim;
    if (n <= 0) {
        if (a.mode != ATTN_OP) pdl_wait();
        if (s == 0 && tid < kHeadDim) outp[tid] = 0.0f;
        return;
    }
    const int ntiles = (n + kAttnTile - 1) / kAttnTile;
    // a row's split boundaries depend only on its own length when tps is fixed, which
    // keeps every row's summation order independent of the rest of the batch
    const int tps = a.tps > 0 ? a.tps : (ntiles + a.S - 1) / a.S;
    const int active = (ntiles + tps - 1) / tps;
    const int t0 = s * tps;
    const int t1 = min(ntiles, t0 + tps);
    if (t0 >= t1) return;

    // grouped-query attention: query head h reads the K/V of head h / kv_group
    const int hk = a.kv_group > 1 ? h / a.kv_group : h;
    const float* Kb = a.k + slot * a.slot_stride + static_cast<long long>(hk) * a.ld * kHeadDim;
    const float* Vb = a.v + slot * a.slot_stride + static_cast<long long>(hk) * a.ld * kHeadDim;

    // tiles before the first one holding a row this step writes can be fetched before the
    // dependency wait (a prompt chunk writes rows fresh..len of its slot in one step)
    const int first_new_tile = (a.mode == ATTN_SELF) ? a.meta->fresh[b] / kAttnTile : ntiles;
    int pre = 0;
    const bool drop = a.drop_first_copy && s == 0 && h == 0 && b == 0;
    if (tid == 0) {
        for (int i = 0; i < NS; ++i) mbar_init(&bars[i], 1);
        mbar_fence_init();
        for (; pre < NS && t0 + pre < t1 && t0 + pre < first_new_tile; ++pre)
            attn_issue(sK + pre * kAttnTile * kHeadDim, sV + pre * kAttnTile * kHeadDim, &bars[pre], a, Kb, Vb,
                       slot, hk, t0 + pre, n, drop && pre == 0);
    }
    pdl_launch_dependents();
    if (a.mode != ATTN_OP) pdl_wait();
    if (tid < kHeadDim) sq[tid] = a.q[b * a.q_bstride + h * kHeadDim + tid];
    if (tid == 0) {
        for (int i = pre; i < NS && t0 + i < t1; ++i)
            attn_issue(sK + i * kAttnTile * kHeadDim, sV + i * kAttnTile * kHeadDim, &bars[i], a, Kb, Vb, slot,
                       hk, t0 + i, n, drop && i == 0);
    }
    __syncthreads();

    const int jj = lane & 15, half = lane >> 4;
    const int key_in_tile = warp * 16 + jj;
    float m = -INFINITY, l = 0.0f, o0 = 0.0f, o1 = 0.0f;

    for (int t = t0; t < t1; ++t) {
        const int it = t - t0;
        const int stage = it % NS;
        const uint32_t phase = static_cast<uint32_t>(it / NS) & 1u;
        if (tid == 0) s_flag = mbar_wait_bounded(&bars[stage], phase, a.err) ? 1 : 0;
        __syncthreads();
        if (!s_flag) {
            // Give the copies still in flight a bounded chance to land, then stop reading
            // tiles. The CTA still merges and arrives below, so the row's arrival count
            // returns to zero for the next launch; the status word already says that this
            // launch's output is not valid.
            if (tid == 0) {
                for (int t2 = t; t2 < min(t1, t + NS); ++t2) {
                    const int it2 = t2 - t0;
                    mbar_wait_bounded(&bars[it2 % NS], static_cast<uint32_t>(it2 / NS) & 1u, nullptr);
                }
            }
            __syncthreads();
            break;
        }
        // the phase is complete; each thread observes it itself (acquire of the bulk writes)
        if (tid != 0) (void)mbar_try_wait(&bars[stage], phase);
        const float* tK = sK + stage * kAttnTile * kHeadDim;
        const float* tV = sV + stage * kAttnTile * kHeadDim;
        const int nvalid = min(kAttnTile, n - t * kAttnTile);

        // score of key `key_in_tile`: this lane's 32 dims, rotated by jj so the 8
        // lanes of a quarter-warp hit 8 different 16-byte bank groups
        const float* krow = tK + key_in_tile * kHeadDim + half * 32;
        const float* qh = sq + half * 32;
        float part = 0.0f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int cc = (c + jj) & 7;
            const float4 kv = *reinterpret_cast<const float4*>(krow + cc * 4);
            const float4 qv = *reinterpret_cast<const float4*>(qh + cc * 4);
            part = fmaf(kv.x, qv.x, part);
            part = fmaf(kv.y, qv.y, part);
            part = fmaf(kv.z, qv.z, part);
            part = fmaf(kv.w, qv.w, part);
        }
        part += __shfl_xor_sync(0xffffffffu, part, 16);
        const bool valid = key_in_tile < nvalid;
        const float sc = valid ? part * 0.125f : -INFINITY;
        const int wvalid = max(0, min(16, nvalid - warp * 16));
        if (wvalid > 0) {
            float tmax = sc;
#pragma unroll
            for (int off = 8; off >= 1; off >>= 1)
                tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
            const float mnew = fmaxf(m, tmax);
            const float corr = expf(m - mnew);
            const float p = valid ? expf(sc - mnew) : 0.0f;
            float psum = p;
#pragma unroll
            for (int off = 8; off >= 1; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
            l = l * corr + psum;
            o0 *= corr;
            o1 *= corr;
            const float* vcol = tV + warp * 16 * kHeadDim + 2 * lane;
            for (int j = 0; j < wvalid; ++j) {
                const float pj = __shfl_sync(0xffffffffu, p, j);
                const float2 vv = *reinterpret_cast<const float2*>(vcol + j * kHeadDim);
                o0 = fmaf(pj, vv.x, o0);
                o1 = fmaf(pj, vv.y, o1);
            }
            m = mnew;
        }
        __syncthreads();
        if (tid == 0 && t + NS < t1)
            attn_issue(sK + stage * kAttnTile * kHeadDim, sV + stage * kAttnTile * kHeadDim, &bars[stage], a, Kb, Vb,
                       slot, hk, t + NS, n);
    }

    // merge the four warps
    if (lane == 0) {
        wm[warp] = m;
        wl[warp] = l;
    }
    wo[warp][2 * lane] = o0;
    wo[warp][2 * lane + 1] = o1;
    __syncthreads();
    float M = -INFINITY, L = 0.0f, oc = 0.0f;
    if (tid < kHeadDim) {
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, wm[w]);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const float e = (wm[w] == -INFINITY) ? 0.0f : expf(wm[w] - M);
            L = fmaf(e, wl[w], L);
            oc = fmaf(e, wo[w][tid], oc);
        }
    }
    if (active == 1) {
        if (tid < kHeadDim) outp[tid] = (L > 0.0f && isfinite(L)) ? oc / L : 0.0f;
        return;
    }
    float* mypart = a.part + ((static_cast<long long>(b) * a.H + h) * a.S + s) * kAttnPartStride;
    if (tid < kHeadDim) mypart[4 + tid] = oc;
    if (tid == 0) {
        mypart[0] = M;
        mypart[1] = L;
    }
    __syncthreads();
    __shared__ int s_last;
    if (tid == 0) {
        __threadfence();
        const int prev = atomicAdd(&a.counters[b * a.H + h], 1);
        s_last = (prev == active - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const float* base = a.part + (static_cast<long long>(b) * a.H + h) * a.S * kAttnPartStride;
    // the split maxima and sums are fetched in parallel (one thread each, at most 32
    // splits), then every output dim sums the splits in split order
    __shared__ float pm[32], pl[32], pw[32];
    if (tid < active) {
        pm[tid] = __ldcg(base + tid * kAttnPartStride);
        pl[tid] = __ldcg(base + tid * kAttnPartStride + 1);
    }
    __syncthreads();
    float M2 = -INFINITY;
    for (int i = 0; i < active; ++i) M2 = fmaxf(M2, pm[i]);
    if (tid < active) pw[tid] = (pm[tid] == -INFINITY) ? 0.0f : expf(pm[tid] - M2);
    __syncthreads();
    if (tid < kHeadDim) {
        float L2 = 0.0f, o = 0.0f;
#pragma unroll 8
        for (int i = 0; i < active; ++i) {
            L2 = fmaf(pw[i], pl[i], L2);
            o = fmaf(pw[i], __ldcg(base + i * kAttnPartStride + 4 + tid), o);
        }
        outp[tid] = (L2 > 0.0f && isfinite(L2)) ? o / L2 : 0.0f;
    }
    if (tid == 0) a.counters[b * a.H + h] = 0;
}

}  // namespace dec
