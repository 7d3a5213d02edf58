// Device helpers shared by the decoder kernels (sm_100a).
#pragma once

#include <cuda.h>

#include <cuda_runtime.h>
#include <stdint.h>

#define DEC_DEVERR_TIMEOUT 1

namespace dec {

constexpr int kHeadDim = 64;
constexpr int kMaxBatch = 128;
// A bounded device wait gives up after this many nanoseconds and reports DEC_ETIMEOUT.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

// Where self-attention K/V rows live. Row `row` of K/V head `hh` of stream slot `slot` starts at
// float offset ((page * heads + hh) * page_rows + r) * 64 of a layer's cache. A paged cache
// (16, 32 or 64 rows per page) takes page = table[slot * pages_per_slot + row / page_rows] and
// r = row % page_rows; a dense cache is the same layout with one page per slot (page = slot,
// page_rows = the slot's rows, r = row).
struct KvMap {
    const int* table;     // paged: physical page of each (slot, logical page); null: dense
    int page_rows;
    int pages_per_slot;
    int heads;            // K/V heads
};

__host__ __device__ __forceinline__ long long kv_page_off(const KvMap& m, int page, int hh, int r) {
    return ((static_cast<long long>(page) * m.heads + hh) * m.page_rows + r) * kHeadDim;
}
__device__ __forceinline__ void kv_page_of(const KvMap& m, int slot, int row, int& page, int& r) {
    if (m.table) {
        page = m.table[slot * m.pages_per_slot + row / m.page_rows];
        r = row % m.page_rows;
    } else {
        page = slot;
        r = row;
    }
}

// Page-table entries a step writes before any kernel reads them (paged caches): the first
// kernel of the step applies them.
constexpr int kMaxTableUpdates = 256;

// Per-step description of the batch, uploaded once per step and read by every kernel.
struct StepMeta {
    int B;
    int pad_[3];
    int slot[kMaxBatch];   // cache slot of batch row b
    int tok[kMaxBatch];    // input token, or -1 for the slot's previous greedy pick
    int pos[kMaxBatch];    // learned-position row / RoPE position
    int len[kMaxBatch];    // cached rows before this step; the new row goes here
    int fresh[kMaxBatch];  // first cache row of the row's slot that this step writes (len, or the
                           // chunk's first row when several rows of one slot run together)
    int n_upd;             // page-table updates: table[upd_idx[i]] = upd_page[i]
    int upd_idx[kMaxTableUpdates];
    int upd_page[kMaxTableUpdates];
};

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier + bulk async copy (global -> shared, no multicast) ----------------

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// 1-D bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// 2-D tiled TMA load (no multicast) of the box at (x, y) of `map` into shared memory,
// completing on `bar`. x times the element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(phase)
        : "memory");
    return ok != 0;
}

// Device status block of a handle: word 0 is the status (DEC_DEVERR_* bits), words 2-3 the
// wait limit in nanoseconds as an unsigned 64-bit value (0: kWaitLimitNs).
constexpr int kStatusWords = 4;

__device__ __forceinline__ unsigned long long wait_limit_ns(const int* err) {
    if (err == nullptr) return kWaitLimitNs;
    const unsigned long long v = *reinterpret_cast<const volatile unsigned long long*>(err + 2);
    return v ? v : kWaitLimitNs;
}

// Wait for phase `phase` of `bar`, giving up after the status block's wait limit (kWaitLimitNs
// without one). On give-up the status word gets DEC_DEVERR_TIMEOUT and false is returned.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t phase, int* err) {
    if (mbar_try_wait(bar, phase)) return true;
    const unsigned long long t0 = global_ns();
    const unsigned long long limit = wait_limit_ns(err);
    while (true) {
        if (mbar_try_wait(bar, phase)) return true;
        if (global_ns() - t0 > limit) {
            if (err) atomicOr(err, DEC_DEVERR_TIMEOUT);
            return false;
        }
    }
}

// ---- launch attributes --------------------------------------------------------------

// Every kernel of the step prefers the largest shared-memory carveout, so that consecutive
// kernels never need the SM's L1 / shared-memory split changed between them: a change
// drains the SM first, which stops a dependent kernel's CTAs from starting early under
// programmatic dependent launch. Applied once per kernel and device (`attr_dev` is the
// caller's per-kernel record of the device it was last applied on).
// max_dyn_smem > 0 also raises the kernel's dynamic shared-memory limit to that many bytes.
template <typename K>
inline cudaError_t prefer_max_shared_once(K kern, int& attr_dev, int max_dyn_smem = 0) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || attr_dev == dev) return e;
    if (max_dyn_smem > 0) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dyn_smem);
        if (e != cudaSuccess) return e;
    }
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess) attr_dev = dev;
    return e;
}

// ---- programmatic dependent launch -----------------------------------------------

__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- warp reductions ---------------------------------------------------------------

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Reduce N per-lane partial values across the warp so that value index i ends up
// summed in lane i << (5 - log2 N) (lanes in between hold copies). N is a power of
// two <= 32. Each halving step exchanges half of the live values with the partner
// lane, so the whole reduction costs N - 1 + (5 - log2 N) shuffles instead of 5 N.
template <int N, typename T>
__device__ __forceinline__ T warp_reduce_transpose(T (&v)[N]) {
    static_assert((N & (N - 1)) == 0 && N >= 1 && N <= 32, "N must be a power of two <= 32");
    const int lane = threadIdx.x & 31;
    int live = N;
    // Exchange halves while more than one value is live.
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        if (live > 1) {
            const int h = live >> 1;
            const bool upper = (lane & off) != 0;
#pragma unroll
            for (int j = 0; j < (N > 1 ? N / 2 : 1); ++j) {
                if (j < h) {
                    T send = upper ? v[j] : v[j + h];
                    T keep = upper ? v[j + h] : v[j];
                    v[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
            }
            live = h;
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
        }
    }
    return v[0];
}

// Lane i holds value index (i >> shift) after warp_reduce_transpose<N>.
template <int N>
__device__ __forceinline__ constexpr int transpose_shift() {
    return N == 32 ? 0 : N == 16 ? 1 : N == 8 ? 2 : N == 4 ? 3 : N == 2 ? 4 : 5;
}

// Orderable 64-bit key for the greedy argmax: larger value wins, lower index wins
// ties; NaN never wins.
__device__ __forceinline__ unsigned long long argmax_key(float v, int idx) {
    if (v != v) return 0ull;
    uint32_t u = __float_as_uint(v);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return (static_cast<unsigned long long>(u) << 32) |
           static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(idx));
}
__device__ __forceinline__ int argmax_key_index(unsigned long long k) {
    return static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(k & 0xFFFFFFFFull));
}

__device__ __forceinline__ float gelu_tanh_f(float x) {
    // 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))
    const float k0 = 0.7978845608028654f;
    const float x3 = x * x * x;
    return 0.5f * x * (1.0f + tanhf(k0 * (x + 0.044715f * x3)));
}

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + expf(-x)); }

}  // namespace dec
