// Launch planning for the projection kernels (batch tile, K chunk, pipeline depth,
// grid size). The template is instantiated explicitly in gemv_inst_*.cu so the many
// variants compile in parallel; other translation units only see the declaration.
#pragma once

#include <cuda_runtime.h>

#include <algorithm>

#include "gemv.cuh"

namespace dec {

constexpr size_t kGemvXBudget = 128 * 1024;      // activation tile bytes at most
constexpr size_t kGemvRingBudget = 48 * 1024;    // weight ring bytes
constexpr size_t kGemvSmemMax = 227 * 1024;

template <typename WT, bool I8, int PRO, int EPI, int MAP>
cudaError_t gemv_launch(int num_sms, const GemvArgs& a, cudaStream_t st);

#ifdef DEC_GEMV_DEFINE

struct GemvPlan {
    int KC, NS;
    size_t smem;
};

// Activation bytes in shared memory: the tile, plus the raw f32 rows for the int8 path,
// plus the norm's weight (and LayerNorm bias) rows.
template <bool I8, int PRO>
size_t gemv_xbytes(int BT, int K) {
    size_t x = size_t(BT) * K * (I8 ? 1 : 4);
    if (I8 && PRO != PRO_RAW_I8) x += size_t(BT) * K * 4;
    if (PRO == PRO_RMS || PRO == PRO_LN) x += size_t(K) * 4;
    if (PRO == PRO_LN) x += size_t(K) * 4;
    return x;
}

template <typename WT, bool I8, int PRO>
GemvPlan gemv_plan(int BT, int K) {
    GemvPlan p;
    const int elt_w = sizeof(WT);
    const int rows_per_block = gemv_rows_per_task(BT) * gemv_consumer_warps(BT);
    // one stage = rows_per_block rows x KC columns (whole rows when they fit)
    int kc = gemv_stage_bytes(BT) / (rows_per_block * elt_w);
    kc = std::min(kc, K);
    kc = std::max(16, kc / 16 * 16);
    p.KC = kc;
    const size_t stage = size_t(rows_per_block) * kc * elt_w;
    const size_t xbytes = gemv_xbytes<I8, PRO>(BT, K);
    // two CTAs per SM when the activation tile leaves room for two stages each,
    // otherwise one CTA with a deeper ring
    const size_t two_cta = 110 * 1024;
    size_t ring;
    if (xbytes + 2 * stage <= two_cta)
        ring = two_cta - xbytes;
    else
        ring = 220 * 1024 - xbytes;
    p.NS = int(std::min<size_t>(kGemvMaxStages, std::max<size_t>(2, ring / stage)));
    p.smem = size_t(p.NS) * stage + xbytes;
    return p;
}

template <int BT, typename WT, bool I8, int PRO, int EPI, int MAP>
cudaError_t gemv_launch_bt(int num_sms, const GemvArgs& a, cudaStream_t st) {
    auto kern = k_gemv<BT, WT, I8, PRO, EPI, MAP>;
    const GemvPlan p = gemv_plan<WT, I8, PRO>(BT, a.K);
    thread_local int attr_dev = -1;   // attributes are per device; set again when it changes
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (attr_dev != dev) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kGemvSmemMax - 2048));
        if (e != cudaSuccess) return e;
        // one shared-memory carveout for every kernel of the step, so that consecutive
        // kernels can share an SM without reconfiguring it
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        attr_dev = dev;
    }
    const int n_pairs = (MAP == MAP_DUAL) ? a.N : (a.N + 1) / 2;
    const int pairs_per_task = gemv_rows_per_task(BT) / 2;
    const int n_tasks = (n_pairs + pairs_per_task - 1) / pairs_per_task;
    const int n_blocks = (n_tasks + gemv_consumer_warps(BT) - 1) / gemv_consumer_warps(BT);
    // occupancy for this instantiation, cached per shared-memory size (per thread)
    thread_local size_t occ_smem[8] = {~size_t(0), ~size_t(0), ~size_t(0), ~size_t(0),
                                 ~size_t(0), ~size_t(0), ~size_t(0), ~size_t(0)};
    thread_local int occ_val[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    thread_local int occ_next = 0;
    auto occupancy = [&](size_t smem, int* occ) -> cudaError_t {
        for (int i = 0; i < 8; ++i)
            if (occ_smem[i] == smem) {
                *occ = occ_val[i];
                return cudaSuccess;
            }
        const cudaError_t r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(occ, kern, gemv_threads(BT), smem);
        if (r != cudaSuccess) return r;
        occ_smem[occ_next] = smem;
        occ_val[occ_next] = *occ;
        occ_next = (occ_next + 1) & 7;
        return cudaSuccess;
    };
    // The ring holds no more stages than a CTA streams, so a small matrix leaves shared
    // memory free and the next kernel's CTAs can become resident early and prefetch
    // their weights while this one runs (programmatic dependent launch).
    const int gy = (a.B + BT - 1) / BT;
    const int elt_w = sizeof(WT);
    const int rows_per_block = gemv_rows_per_task(BT) * gemv_consumer_warps(BT);
    const size_t stage = size_t(rows_per_block) * p.KC * elt_w;
    const size_t xbytes = p.smem - size_t(p.NS) * stage;
    const int chunks = (a.K + p.KC - 1) / p.KC;
    int occ = 0, gx = 1, ns = p.NS;
    for (int pass = 0; pass < 2; ++pass) {
        e = occupancy(xbytes + size_t(pass == 0 ? 2 : ns) * stage, &occ);
        if (e != cudaSuccess) return e;
        gx = std::max(1, std::min(n_blocks, (num_sms * std::max(1, occ)) / gy));
        const int items = ((n_blocks + gx - 1) / gx) * chunks;
        ns = std::min(p.NS, std::max(2, items));
    }
    const size_t smem = xbytes + size_t(ns) * stage;
    // one wave at the final ring depth
    e = occupancy(smem, &occ);
    if (e != cudaSuccess) return e;
    gx = std::max(1, std::min(gx, (num_sms * std::max(1, occ)) / gy));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(gx, gy);
    cfg.blockDim = dim3(gemv_threads(BT));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a, p.KC, ns);
}

template <typename WT, bool I8, int PRO, int EPI, int MAP>
cudaError_t gemv_launch(int num_sms, const GemvArgs& a, cudaStream_t st) {
    // batch tile: the largest power of two <= 32 covering the batch whose activation
    // tile fits the budget
    int bt = 1;
    while (bt < a.B && bt < 32) bt <<= 1;
    while (bt > 1 && gemv_xbytes<I8, PRO>(bt, a.K) > kGemvXBudget) bt >>= 1;
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
