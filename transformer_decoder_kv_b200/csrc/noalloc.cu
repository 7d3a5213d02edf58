// dec_attention_noalloc: split-K decode attention whose scratch (partial softmax
// states and arrival counters) is a fixed array in this library instead of a
// caller-provided workspace. For callers that cannot allocate device memory.

#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "../../include/dec.h"
#include "attention.cuh"

void dec_set_thread_error(const char* msg);

namespace {

constexpr int kNoAllocMaxRows = 1024;   // batch * n_heads
constexpr int kNoAllocMaxSplits = 8;
constexpr size_t kCounterBytes = size_t(kNoAllocMaxRows) * sizeof(int);   // 4 KB, 256-aligned
constexpr size_t kPartBytes = size_t(kNoAllocMaxRows) * kNoAllocMaxSplits * dec::kAttnPartStride * sizeof(float);
constexpr size_t kScratchBytes = kCounterBytes + kPartBytes;
constexpr int kMaxDevices = 64;

}  // namespace

// The scratch: counters [1024] int32, then partial states [1024][8][68] f32. In host
// code this name is only a stand-in; the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_attn_noalloc_scratch[kScratchBytes];

namespace {

std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDevices] = {};

dec_status fail(dec_status st, const std::string& msg) {
    dec_set_thread_error(msg.c_str());
    return st;
}

// Once per device, with that device current: the array's device address, and the
// kernel's shared-memory opt-in.
dec_status setup(int dev, void** addr) {
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_attn_noalloc_scratch);
        if (e != cudaSuccess) return fail(DEC_ECUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
        e = cudaFuncSetAttribute(dec::k_attention, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(dec::kAttnSmemBytes));
        if (e != cudaSuccess) return fail(DEC_ECUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return DEC_OK;
}

// Split count: fewest waves x tiles per CTA, at most kNoAllocMaxSplits.
int splits_for(int num_sms, int rows, int max_tiles) {
    if (max_tiles <= 1) return 1;
    const int slots = num_sms * 2;
    int best = 1;
    double best_cost = 1e30;
    for (int s = 1; s <= (max_tiles < kNoAllocMaxSplits ? max_tiles : kNoAllocMaxSplits); ++s) {
        const int tps = (max_tiles + s - 1) / s;
        if ((max_tiles + tps - 1) / tps != s) continue;
        const double waves = double((rows * s + slots - 1) / slots);
        const double cost = waves * (tps + 1.5) + (s > 1 ? 0.5 : 0.0);
        if (cost < best_cost) {
            best_cost = cost;
            best = s;
        }
    }
    return best;
}

}  // namespace

extern "C" dec_status dec_attention_noalloc(const float* q, const float* k, const float* v, const int32_t* lens,
                                            int32_t batch, int32_t n_heads, int32_t ld, float* out,
                                            void* stream) {
    if (!q || !k || !v || !lens || !out) return fail(DEC_EINVAL, "dec_attention_noalloc: null pointer");
    if (batch < 1 || n_heads < 1 || ld < 1) return fail(DEC_EINVAL, "dec_attention_noalloc: bad shape");
    if (static_cast<long long>(batch) * n_heads > kNoAllocMaxRows)
        return fail(DEC_EINVAL, "dec_attention_noalloc: batch * n_heads = " +
                                    std::to_string(static_cast<long long>(batch) * n_heads) +
                                    " exceeds the fixed scratch limit of " + std::to_string(kNoAllocMaxRows));
    if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15)
        return fail(DEC_EINVAL, "dec_attention_noalloc: k and v must be 16-byte aligned");
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(DEC_ECUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(DEC_EINVAL, "dec_attention_noalloc: device index too large");
    void* base = nullptr;
    dec_status st = setup(dev, &base);
    if (st != DEC_OK) return st;
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the arrival counters must start at zero
    e = cudaMemsetAsync(base, 0, size_t(batch) * n_heads * sizeof(int), s);
    if (e != cudaSuccess) return fail(DEC_ECUDA, std::string("cudaMemsetAsync: ") + cudaGetErrorString(e));
    dec::AttnArgs a{};
    a.q = q;
    a.q_bstride = static_cast<long long>(n_heads) * dec::kHeadDim;
    a.k = k;
    a.v = v;
    a.slot_stride = static_cast<long long>(n_heads) * ld * dec::kHeadDim;
    a.ld = ld;
    a.H = n_heads;
    a.mode = dec::ATTN_OP;
    a.batch = batch;
    a.lens = lens;
    a.out = out;
    a.out_bstride = static_cast<long long>(n_heads) * dec::kHeadDim;
    a.counters = static_cast<int*>(base);
    a.part = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + kCounterBytes);
    a.err = nullptr;
    a.S = splits_for(sms, batch * n_heads, (ld + dec::kAttnTile - 1) / dec::kAttnTile);
    dec::k_attention<<<dim3(a.S, n_heads, batch), dec::kAttnThreads, dec::kAttnSmemBytes, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(DEC_ECUDA, std::string("k_attention launch: ") + cudaGetErrorString(e));
    return DEC_OK;
}
