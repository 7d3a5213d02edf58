// Launch planning for the projection kernels (batch tile, K chunking, grid size).
// The template is instantiated explicitly in gemv_inst_*.cu so the many variants
// compile in parallel; other translation units only see the declaration.
#pragma once

#include <cuda_runtime.h>

#include <algorithm>

#include "gemv.cuh"

namespace dec {

constexpr size_t kGemvSmemBudget = 96 * 1024;

template <typename WT, bool I8, int PRO, int EPI, int MAP>
cudaError_t gemv_launch(int num_sms, const GemvArgs& a, cudaStream_t st);

#ifdef DEC_GEMV_DEFINE

inline int gemv_pow2ceil(int v) {
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

template <int BT, typename WT, bool I8, int PRO, int EPI, int MAP>
cudaError_t gemv_launch_bt(int num_sms, const GemvArgs& a, cudaStream_t st) {
    auto kern = k_gemv<BT, WT, I8, PRO, EPI, MAP>;
    const size_t elt = I8 ? 1 : 4;
    int KC = a.K;
    if (size_t(BT) * a.K * elt > kGemvSmemBudget) {
        KC = int(kGemvSmemBudget / (size_t(BT) * elt));
        KC = std::max(64, KC / 64 * 64);
    }
    const size_t smem = size_t(BT) * KC * elt;
    static int per_sm = 0;  // per instantiation: occupancy at the full budget
    cudaError_t e;
    if (per_sm == 0) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kGemvSmemBudget));
        if (e != cudaSuccess) return e;
        per_sm = -1;
    }
    const int n_tasks = (MAP == MAP_DUAL) ? a.N : (a.N + 1) / 2;
    const int need = (n_tasks + kGemvWarps - 1) / kGemvWarps;
    int gx = need;
    if (KC == a.K) {
        // occupancy for this instantiation, cached per activation-tile size
        static size_t occ_smem[4] = {~size_t(0), ~size_t(0), ~size_t(0), ~size_t(0)};
        static int occ_val[4] = {0, 0, 0, 0};
        int occ = -1;
        for (int i = 0; i < 4; ++i)
            if (occ_smem[i] == smem) occ = occ_val[i];
        if (occ < 0) {
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kGemvThreads, smem);
            if (e != cudaSuccess) return e;
            static int next = 0;
            occ_smem[next] = smem;
            occ_val[next] = occ;
            next = (next + 1) & 3;
        }
        gx = std::min(need, num_sms * std::max(1, occ));
    }
    const int gy = (a.B + BT - 1) / BT;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(gx, gy);
    cfg.blockDim = dim3(kGemvThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a, KC);
}

template <typename WT, bool I8, int PRO, int EPI, int MAP>
cudaError_t gemv_launch(int num_sms, const GemvArgs& a, cudaStream_t st) {
    const int bt = std::min(32, gemv_pow2ceil(a.B));
    switch (bt) {
        case 1: return gemv_launch_bt<1, WT, I8, PRO, EPI, MAP>(num_sms, a, st);
        case 2: return gemv_launch_bt<2, WT, I8, PRO, EPI, MAP>(num_sms, a, st);
        case 4: return gemv_launch_bt<4, WT, I8, PRO, EPI, MAP>(num_sms, a, st);
        case 8: return gemv_launch_bt<8, WT, I8, PRO, EPI, MAP>(num_sms, a, st);
        case 16: return gemv_launch_bt<16, WT, I8, PRO, EPI, MAP>(num_sms, a, st);
        default: return gemv_launch_bt<32, WT, I8, PRO, EPI, MAP>(num_sms, a, st);
    }
}

#define DEC_GEMV_INSTANTIATE(WT, I8, PRO, EPI, MAP) \
    template cudaError_t gemv_launch<WT, I8, PRO, EPI, MAP>(int, const GemvArgs&, cudaStream_t);

#endif  // DEC_GEMV_DEFINE

}  // namespace dec
