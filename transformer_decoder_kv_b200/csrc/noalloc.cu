// dec_attention_noalloc: split-K decode attention whose scratch (partial softmax
// states and arrival counters) is a fixed array in this library instead of a
// caller-provided workspace. For callers that cannot allocate device memory.

#include <cuda_runtime.h>

#include <string>

#include "../../include/dec.h"
#include "attn_plan.h"

void dec_set_thread_error(const char* msg);

namespace {

constexpr int kNoAllocMaxRows = 1024;   // batch * n_heads
constexpr int kNoAllocMaxSplits = dec::kAttnMaxSplits;   // the same split cap as dec_attention
constexpr size_t kStatusBytes = 256;    // device status word, padded to the array's alignment
constexpr size_t kCounterBytes = size_t(kNoAllocMaxRows) * sizeof(int);   // 4 KB, 256-aligned
constexpr size_t kPartBytes = size_t(kNoAllocMaxRows) * kNoAllocMaxSplits * dec::kAttnPartStride * sizeof(float);
constexpr size_t kScratchBytes = kStatusBytes + kCounterBytes + kPartBytes;

}  // namespace

// The scratch: a status word (padded to 256 bytes), arrival counters [1024] int32, then
// partial states [1024][32][68] f32 -- about 8.9 MB. In host code this name is only a
// stand-in; the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_attn_noalloc_scratch[kScratchBytes];

namespace {

dec_status fail(dec_status st, const std::string& msg) {
    dec_set_thread_error(msg.c_str());
    return st;
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
    // The array's device address on the current device, looked up on every call (cheap once
    // the module is loaded, and valid again after a device reset reloads it), and the
    // kernel's shared-memory opt-in, which is per device as well.
    void* base = nullptr;
    e = cudaGetSymbolAddress(&base, g_attn_noalloc_scratch);
    if (e != cudaSuccess) return fail(DEC_ECUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    e = cudaFuncSetAttribute(dec::k_attention, cudaFuncAttributeMaxDynamicSharedMemorySize, int(dec::kAttnSmemBytes));
    if (e != cudaSuccess) return fail(DEC_ECUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
    int sms = 148;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return fail(DEC_ECUDA, std::string("cudaDeviceGetAttribute: ") + cudaGetErrorString(e));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the status word and the arrival counters must start at zero
    e = cudaMemsetAsync(base, 0, kStatusBytes + size_t(batch) * n_heads * sizeof(int), s);
    if (e != cudaSuccess) return fail(DEC_ECUDA, std::string("cudaMemsetAsync: ") + cudaGetErrorString(e));
    unsigned char* arr = static_cast<unsigned char*>(base);
    // the launch dec_attention makes for the same arguments with tiles_per_split = 0
    const dec::AttnLaunch p = dec::attn_launch_plan(sms, batch * n_heads, ld, 0);
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
    a.err = reinterpret_cast<int*>(arr);
    a.counters = reinterpret_cast<int*>(arr + kStatusBytes);
    a.part = reinterpret_cast<float*>(arr + kStatusBytes + kCounterBytes);
    a.S = p.S;
    a.tps = p.tps;
    a.stages = p.stages;
    dec::k_attention<<<dim3(a.S, n_heads, batch), dec::kAttnThreads, dec::attn_smem_bytes(p.stages), s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(DEC_ECUDA, std::string("k_attention launch: ") + cudaGetErrorString(e));
    return DEC_OK;
}
