// W8A8 and Whisper W8A32 projections on the 5th-generation tensor cores for batches of 8 or more:
// tcgen05.mma .kind::i8 (M = 128 weight rows, N = 16 or 32 batch columns, K = 32 per
// instruction) with exact int32 accumulation in TMEM.
//
// The activation rows come from k_rowprep_i8, the per-row symmetric quantiser with ties to
// even (franken_ocr decoder_qwen2.rs, quantize_row_i8_te) computed with the CUDA-core
// kernel's arithmetic and reduction order, so the codes, the exact int32 sums and the
// dequantisation y = float(acc) * (a_b * s_n) + bias (decoder_qwen2.rs,
// gemv_i8_bias_prequant) are bit-identical to the dp4a kernel used below batch 8.
//
// CTA (320 threads, one per SM): warp 0 streams 128-row x 128-column weight boxes by TMA
// (no multicast) into a ring of 16 KB stages and loads the CTA's K slice of the activation
// rows once; warp 1 owns the TMEM allocation (two accumulator sets) and issues the MMAs,
// committing each stage back to the producer and each finished row block to the
// epilogue; warps 2..9 read the accumulators with tcgen05.ld. A warp may only touch the
// TMEM lane quarter (warp id mod 4), i.e. 32 weight rows, so two warps share each quarter
// and each finishes one row and half of the batch columns per thread, which halves the
// serial chain of dequantise-and-store work behind the last MMA. A tcgen05.mma .kind::i8 of
// M = 128, K = 32 takes about 135 SM cycles whatever its N (measured on B200 for N = 16 to
// 256, with one or many independent accumulators), so the MMA phase costs one such time per
// instruction: the activation digit planes of a batch tile are stacked along N in shared
// memory, and one instruction multiplies a weight plane by all the planes it pairs with.
// K is split across CTA
// groups so that small matrices still reach every SM; with more than one slice, each
// epilogue warp stores its exact partial sums and the last of the n_ks warps that own a
// 32-row, half-tile group (an arrival count; nothing waits) adds the slices and finishes.
//
// Row maps: the NEOX RoPE pair (i, i + 32) of a head and the SwiGLU pair (gate n, up n) are
// stored in adjacent weight rows (MAP_ROPE: row 2j holds i = j, row 2j + 1 holds i = 32 + j
// in each 64-row head block; MAP_DUAL: row 2n holds gate n, row 2n + 1 up n), so a pair
// sits in adjacent TMEM lanes and meets through one shuffle.
#pragma once

#include "head_tc.cuh"
#include "proj_mma.cuh"
#include "rowprep_i8.cuh"

namespace dec {

constexpr int kTcThreads = 320;                 // producer, MMA issuer, 8 epilogue warps
constexpr int kTcEpiWarps = 8;                  // two per TMEM lane quarter, half the columns each
constexpr int kTcKC = 128;                      // K per stage (one 128-byte box)
constexpr int kTcStageBytes = 128 * kTcKC;      // 16 KB
constexpr int kTcMaxStages = 12;
constexpr int kTcMaxBT = 32;
constexpr size_t kTcXBudget = 120 * 1024;       // activation slice bytes at most (all planes)

struct TcArgs {
    CUtensorMap wmap;      // int8 weight planes [WD * n_rows, K]: box {128 bytes, 128 rows}
    CUtensorMap xmap;      // int8 activation planes [XD * MB, K]: box {128 bytes, BT rows}
    const float* xs;       // [B] activation scales
    int* part;             // split-K partial sums
    int* cnt;              // arrival counts per (row block, batch tile, lane quarter, half), zero between launches
    int n_ks, ksl, n_rows, n_by;
    int MB;                // rows of one activation plane
    GemvArgs g;            // shapes and epilogue arguments
};

// Logical row of physical row p under the tensor-core row maps.
template <int MAP>
__host__ __device__ __forceinline__ int tc_logical_row(int p) {
    if (MAP == MAP_ROPE) {
        const int w = p & 63;
        return (p & ~63) + ((w & 1) ? 32 + (w >> 1) : (w >> 1));
    }
    if (MAP == MAP_DUAL) return p >> 1;   // gate if p is even, up if odd
    return p;
}

// Digit planes of the two operands: XD activation planes and WD weight planes, each an
// int8 matrix; the products summed into accumulator j are those whose weight is 254^-j.
//   XD = 1, WD = 1 (W8A8):   A0 = W X
//   XD = 3, WD = 1 (W8A32):  A0 = W X1, A1 = W X2, A2 = W X3
//   XD = 3, WD = 3 (f32):    A0 = W1 X1, A1 = W1 X2 + W2 X1, A2 = W1 X3 + W2 X2 + W3 X1
// In shared memory the activation planes of each 128-column chunk are stacked along N
// (plane p in rows p BT .. p BT + BT - 1), and the accumulators A0 | A1 | A2 sit side by side
// in TMEM, so W1 [X1; X2; X3] (N = 3 BT) writes all three at once, W2 [X1; X2] (N = 2 BT) adds
// into A1 | A2 and W3 X1 (N = BT) into A2: one, one and three instructions per K step.
template <int XD, int WD>
struct TcDigits {
    static_assert((XD == 1 && WD == 1) || (XD == 3 && (WD == 1 || WD == 3)), "digit planes");
};
// (WD = 3, f32 weights split like the head's embedding, is supported by the kernel but not
// instantiated: it measured slower than the TF32 kernel at the shapes that use f32 weights.)

// TMEM columns of one CTA: `sets` accumulator sets (two when the CTA owns more than one row
// block, so that the epilogue of one overlaps the MMAs of the next) of XD BT columns; at most
// 256, so that two CTAs of consecutive kernels can hold TMEM at once.
__host__ __device__ inline uint32_t tc_tmem_cols(int xd, int bt, int sets) {
    const int need = sets * xd * bt;
    uint32_t t = 32;
    while (t < static_cast<uint32_t>(need)) t <<= 1;
    return t;
}

template <int BT, int EPI, int MAP, int XD, int WD>
__global__ void __launch_bounds__(kTcThreads, 1) k_proj_tc(const __grid_constant__ TcArgs A, int NS) {
    static_assert(BT == 16 || BT == 32, "batch tile");
    static_assert(XD == 1 || (MAP == MAP_ADJ && EPI != EPI_I32 && EPI != EPI_SWIGLU), "digit planes: plain rows");
    (void)sizeof(TcDigits<XD, WD>);
    constexpr int NACC = XD;                              // accumulators A0 .. A(XD-1)
    constexpr int kStage = WD * kTcStageBytes;
    constexpr int XC = XD * BT * 128;                     // bytes of one chunk's stacked planes
    constexpr uint32_t IDESC1 = idesc_i8(XD * BT);        // W1 against every activation plane
    constexpr uint32_t IDESC2 = idesc_i8(2 * BT);         // W2 against X1, X2
    constexpr uint32_t IDESC3 = idesc_i8(BT);             // W3 against X1
    const GemvArgs& a = A.g;

    extern __shared__ unsigned char tc_smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    unsigned char* ring = smem;
    unsigned char* sx = smem + static_cast<size_t>(NS) * kStage;
    __shared__ __align__(8) uint64_t full[kTcMaxStages], empty[kTcMaxStages];
    __shared__ __align__(8) uint64_t tfull[2], tempty[2], bar_x, bar_done;
    __shared__ uint32_t s_tmem;
    __shared__ float s_xs[BT];
    __shared__ int s_pos[BT], s_slot[BT], s_len[BT];   // EPI_QKV: position, cache page, row in the page
    __shared__ int s_fail;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_by = A.n_by;
    const int by = blockIdx.x % n_by, b0 = by * BT;
    const int nb = min(BT, a.B - b0);
    const int n_blocks = (A.n_rows + 127) / 128;
    const int rest = blockIdx.x / n_by;
    const int ks = rest % A.n_ks;
    const int cps = gridDim.x / (A.n_ks * n_by);
    const int c0 = rest / A.n_ks;
    const int kstart = ks * A.ksl;
    const int klen = min(A.ksl, a.K - kstart);
    const int nch = (klen + kTcKC - 1) / kTcKC;
    const int my_blocks = c0 < n_blocks ? (n_blocks - 1 - c0) / cps + 1 : 0;
    const int n_items = my_blocks * nch;
    const int sets = my_blocks > 1 ? 2 : 1;
    const int setc = XD * BT;                            // TMEM columns of one accumulator set
    const uint32_t tcols = tc_tmem_cols(XD, BT, sets);

    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], kTcEpiWarps);
        }
        mbar_init(&bar_x, 1);
        mbar_init(&bar_done, 1);
        mbar_fence_init();
        s_fail = 0;
    }
    if (warp == 1) {
        tmem_alloc(&s_tmem, tcols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = s_tmem;

    // weight stage `it`: the WD planes of one 128-row block and 128 columns of K
    auto issue = [&](int it) {
        const int jb = c0 + (it / nch) * cps;
        const int c = it % nch;
        unsigned char* dst = ring + static_cast<size_t>(it % NS) * kStage;
        mbar_arrive_expect_tx(&full[it % NS], kStage);
#pragma unroll
        for (int p = 0; p < WD; ++p)
            tma_load_2d(dst + p * kTcStageBytes, &A.wmap, kstart + c * kTcKC, p * A.n_rows + jb * 128,
                        &full[it % NS]);
    };
    int n_issued = 0;
    if (warp == 0 && lane == 0)
        for (; n_issued < NS && n_issued < n_items; ++n_issued) issue(n_issued);
    pdl_launch_dependents();
    pdl_wait();
    if (tid < BT) {
        s_xs[tid] = tid < nb ? A.xs[b0 + tid] : 0.0f;
        if (EPI == EPI_QKV) {
            // position, and the cache page and row within it of this step's new row
            int page = 0, r = 0;
            if (tid < nb) kv_page_of(a.kv, a.meta->slot[b0 + tid], a.meta->len[b0 + tid], page, r);
            s_pos[tid] = tid < nb ? a.meta->pos[b0 + tid] : 0;
            s_slot[tid] = page;
            s_len[tid] = r;
        }
    }
    __syncthreads();

    if (warp == 0 && lane == 0) {
        // the activation slice of this batch tile: XD planes, one box per 128 columns
        mbar_arrive_expect_tx(&bar_x, static_cast<uint32_t>(XD * nch) * BT * 128);
        for (int p = 0; p < XD; ++p)
            for (int c = 0; c < nch; ++c)
                tma_load_2d(sx + c * XC + p * BT * 128, &A.xmap, kstart + c * kTcKC, p * A.MB + b0, &bar_x);
        for (int it = n_issued; it < n_items; ++it) {
            if (!mbar_wait_bounded(&empty[it % NS], static_cast<uint32_t>(it / NS - 1) & 1u, a.err)) {
                s_fail = 1;
                break;
            }
            issue(it);
            n_issued = it + 1;
        }
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issuer ----
        bool ok = mbar_wait_bounded(&bar_x, 0, a.err);
        tc_fence_after();
        int it = 0;
        for (int i = 0; ok && i < my_blocks; ++i) {
            const int ab = i & 1;
            if (i >= 2 && !mbar_wait_bounded(&tempty[ab], static_cast<uint32_t>((i >> 1) - 1) & 1u, a.err)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t dset = tbase + static_cast<uint32_t>(ab * setc);
            for (int c = 0; c < nch; ++c, ++it) {
                const int stage = it % NS;
                if (!mbar_wait_bounded(&full[stage], static_cast<uint32_t>(it / NS) & 1u, a.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const unsigned char* st = ring + static_cast<size_t>(stage) * kStage;
#pragma unroll
                for (int s = 0; s < kTcKC / 32; ++s) {
                    const uint32_t first = (c == 0 && s == 0) ? 0u : 1u;
                    const uint64_t w1 = smem_desc_sw128(st) + 2 * s;
                    const uint64_t xs = smem_desc_sw128(sx + c * XC) + 2 * s;
                    umma_i8(dset, w1, xs, IDESC1, first);
                    if (WD == 3) {
                        const uint64_t w2 = smem_desc_sw128(st + kTcStageBytes) + 2 * s,
                                       w3 = smem_desc_sw128(st + 2 * kTcStageBytes) + 2 * s;
                        umma_i8(dset + BT, w2, xs, IDESC2, 1u);
                        umma_i8(dset + 2 * BT, w3, xs, IDESC3, 1u);
                    }
                }
                umma_commit(&empty[stage]);
            }
            if (!ok) break;
            umma_commit(&tfull[ab]);
        }
        if (!ok) s_fail = 1;
        umma_commit(&bar_done);
        mbar_wait_bounded(&bar_done, 0, nullptr);
    } else if (warp >= 2) {
        // ---- epilogue: lane quarter q holds weight rows 32 q .. 32 q + 31; two warps per
        // quarter, each finishing half of the batch columns (c0b .. c0b + HB - 1) ----
        constexpr int HB = BT / 2;
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        const int c0b = half * HB;
        for (int i = 0; i < my_blocks; ++i) {
            const int ab = i & 1;
            if (!mbar_wait_bounded(&tfull[ab], static_cast<uint32_t>(i >> 1) & 1u, a.err)) {
                s_fail = 1;
                break;
            }
            tc_fence_after();
            int acc[NACC][HB];
            const uint32_t tq = tbase + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(ab * setc + c0b);
#pragma unroll
            for (int j = 0; j < NACC; ++j) HeadTmemLd<HB>::run(tq + static_cast<uint32_t>(j * BT), acc[j]);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[ab]);
            const int jb = c0 + i * cps;
            if (A.n_ks > 1) {
                // exact partial sums of this slice: each thread's NACC x HB values contiguous
                constexpr int NV = NACC * HB;
                const long long grp = ((static_cast<long long>(jb) * n_by + by) * 4 + q) * 2 + half;
                int4* mine = reinterpret_cast<int4*>(A.part + ((grp * A.n_ks + ks) * 32 + lane) * NV);
#pragma unroll
                for (int j = 0; j < NACC; ++j)
#pragma unroll
                    for (int v = 0; v < HB / 4; ++v)
                        mine[j * (HB / 4) + v] =
                            make_int4(acc[j][4 * v], acc[j][4 * v + 1], acc[j][4 * v + 2], acc[j][4 * v + 3]);
                __threadfence();
                __syncwarp();
                int last = 0;
                if (lane == 0) last = (atomicAdd(A.cnt + grp, 1) == A.n_ks - 1);
                last = __shfl_sync(0xffffffffu, last, 0);
                if (!last) continue;
                __threadfence();
#pragma unroll
                for (int j = 0; j < NACC; ++j)
#pragma unroll
                    for (int b = 0; b < HB; ++b) acc[j][b] = 0;
                for (int sl = 0; sl < A.n_ks; ++sl) {
                    const int4* src = reinterpret_cast<const int4*>(A.part + ((grp * A.n_ks + sl) * 32 + lane) * NV);
                    int4 v4[NV / 4];
#pragma unroll
                    for (int v = 0; v < NV / 4; ++v) v4[v] = __ldcg(src + v);
#pragma unroll
                    for (int j = 0; j < NACC; ++j)
#pragma unroll
                        for (int v = 0; v < HB / 4; ++v) {
                            acc[j][4 * v] += v4[j * (HB / 4) + v].x;
                            acc[j][4 * v + 1] += v4[j * (HB / 4) + v].y;
                            acc[j][4 * v + 2] += v4[j * (HB / 4) + v].z;
                            acc[j][4 * v + 3] += v4[j * (HB / 4) + v].w;
                        }
                }
                if (lane == 0) A.cnt[grp] = 0;
            }
            // ---- dequantise and finish row p for this warp's batch columns ----
            // Every global input of the epilogue (row scale, bias, the residual values, the
            // RoPE table entries) is loaded before the first store: a load placed after a
            // store to memory it might alias would wait for that store, one L2 round trip
            // per batch column.
            const int p = jb * 128 + q * 32 + lane;
            const bool row_live = p < A.n_rows;
            const int n = tc_logical_row<MAP>(p);
            const float* sc = (MAP == MAP_DUAL && (p & 1)) ? a.scale2 : a.scale;
            const float sn = row_live ? sc[n] : 0.0f;
            const float bn = (EPI != EPI_SWIGLU && a.bias != nullptr && row_live) ? a.bias[n] : 0.0f;
            int sec = 0, within = n, hh = 0, col = 0;
            if (EPI == EPI_QKV) {
                sec = n < a.d ? 0 : (n < a.d + a.kvd ? 1 : 2);
                within = n - (sec == 0 ? 0 : (sec == 1 ? a.d : a.d + a.kvd));
                hh = within >> 6;
                col = within & 63;
            }
            constexpr bool kRope = EPI == EPI_QKV && MAP == MAP_ROPE;
            float prev[EPI == EPI_RESID ? HB : 1];
            float2 cs[kRope ? HB : 1];
            if (EPI == EPI_RESID) {
#pragma unroll
                for (int j = 0; j < HB; ++j) {
                    const int b = c0b + j;
                    prev[j] = (b < nb && row_live) ? a.out[static_cast<long long>(b0 + b) * a.out_ld + n] : 0.0f;
                }
            }
            if (kRope) {
                const bool rot = a.rope != nullptr && sec < 2 && row_live;
#pragma unroll
                for (int j = 0; j < HB; ++j) {
                    const int b = c0b + j;
                    cs[j] = (rot && b < nb) ? a.rope[static_cast<long long>(s_pos[b]) * 32 + (col & 31)]
                                            : make_float2(1.0f, 0.0f);
                }
            }
            if (EPI == EPI_I32) {
                // the exact int32 sums themselves (kernel-level check of the integer products)
#pragma unroll
                for (int j = 0; j < HB; ++j) {
                    const int b = c0b + j;
                    if (b < nb && row_live) a.out_i32[static_cast<long long>(b0 + b) * a.out_ld + n] = acc[0][j];
                }
                continue;
            }
#pragma unroll
            for (int j = 0; j < HB; ++j) {
                const int b = c0b + j;
                float y;
                if (XD == 1)
                    y = __fmul_rn(static_cast<float>(acc[0][j]), __fmul_rn(s_xs[b], sn));
                else
                    y = digit_logit(acc[0][j], acc[NACC > 1 ? 1 : 0][j], acc[NACC > 2 ? 2 : 0][j], sn, s_xs[b]);
                if (EPI != EPI_SWIGLU && a.bias != nullptr) y = __fadd_rn(y, bn);
                const float yp = __shfl_xor_sync(0xffffffffu, y, 1);   // partner row of a pair
                if (b >= nb || !row_live) continue;
                const int gb = b0 + b;
                if (EPI == EPI_RESID) {
                    a.out[static_cast<long long>(gb) * a.out_ld + n] = __fadd_rn(prev[EPI == EPI_RESID ? j : 0], y);
                } else if (EPI == EPI_SWIGLU) {
                    if ((p & 1) == 0) a.out[static_cast<long long>(gb) * a.out_ld + n] = __fmul_rn(silu_f(y), yp);
                } else if (EPI == EPI_GELU) {
                    a.out[static_cast<long long>(gb) * a.out_ld + n] = gelu_tanh_f(y);
                } else if (EPI == EPI_QKV) {
                    float val = y;
                    if (kRope && a.rope != nullptr && sec < 2) {
                        const float2 c = cs[kRope ? j : 0];
                        // pair (i, i + 32): x_i' = x_i c - x_{i+32} s ; x_{i+32}' = x_i s + x_{i+32} c
                        if (col < 32)
                            val = __fsub_rn(__fmul_rn(y, c.x), __fmul_rn(yp, c.y));
                        else
                            val = __fadd_rn(__fmul_rn(yp, c.y), __fmul_rn(y, c.x));
                    }
                    if (sec == 0) {
                        a.out[static_cast<long long>(gb) * a.out_ld + within] = val;
                    } else {
                        float* cache = (sec == 1) ? a.kc : a.vc;
                        cache[kv_page_off(a.kv, s_slot[b], hh, s_len[b]) + col] = val;
                    }
                } else if (EPI == EPI_STORE) {
                    a.out[static_cast<long long>(gb) * a.out_ld + n] = y;
                }
            }
        }
    }
    if (warp == 0 && lane == 0 && s_fail)
        for (int i2 = max(0, n_issued - NS); i2 < n_issued; ++i2)
            mbar_wait_bounded(&full[i2 % NS], static_cast<uint32_t>(i2 / NS) & 1u, nullptr);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, tcols);
    }
}

// ---------------------------------------------------------------- launch planning

// K split of one projection on tcgen05 with XD activation planes; a function of the shape
// only. A CTA takes whole 128-row blocks over all of K whenever the batch tile's activation
// slice fits: measured on B200 (per-phase timestamps inside the kernel at batch 16 and 64),
// exchanging split-K partials -- partial tiles to global memory, a fence, an arrival count,
// and the last arriver reading every slice -- cost 5-10 us on the critical path, more than
// the parallelism it bought, since the weights are already streamed in during the previous
// kernel. Longer K is split into the fewest slices whose activation slice fits.
inline MmaPlan tc_plan(int n_rows, int K, int num_sms, int xd = 1) {
    (void)num_sms;
    MmaPlan p{};
    p.nbx = 1;
    p.n_blocks = (n_rows + 127) / 128;
    if (K % 32 != 0 || n_rows <= 0) return p;
    const int kchunks = (K + kTcKC - 1) / kTcKC;
    auto slice_len = [&](int nks) { return std::min(((kchunks + nks - 1) / nks) * kTcKC, K); };
    auto xbytes = [&](int len) { return size_t(xd) * kTcMaxBT * ((len + kTcKC - 1) / kTcKC) * 128; };
    int n_ks = 1;
    while (xbytes(slice_len(n_ks)) > kTcXBudget && n_ks < kchunks) ++n_ks;
    p.ksl = slice_len(n_ks);
    p.n_ks = (K + p.ksl - 1) / p.ksl;
    p.ok = xbytes(p.ksl) <= kTcXBudget;
    return p;
}
inline size_t tc_part_bytes(const MmaPlan& p, int B, int xd = 1) {
    const int gy = (B + kTcMaxBT - 1) / kTcMaxBT;
    return p.n_ks > 1 ? size_t(p.n_blocks) * gy * p.n_ks * 128 * kTcMaxBT * 4 * (xd == 3 ? 3 : 1) : 0;
}
inline int tc_counters(const MmaPlan& p, int B) { return p.n_blocks * ((B + kTcMaxBT - 1) / kTcMaxBT) * 4 * 2; }

// One projection on tcgen05: wmap over the WD weight planes, xmap16 / xmap32 over the XD
// activation planes (MB rows each) with boxes of 16 / 32 rows; xs the activation row scales.
template <int EPI, int MAP, int XD, int WD>
cudaError_t proj_tc_launch(int num_sms, const CUtensorMap& wmap, const CUtensorMap& xmap16, const CUtensorMap& xmap32,
                           int n_rows, int MB, const float* xs, void* part, size_t part_bytes, int* cnt, int cnt_len,
                           const GemvArgs& g, cudaStream_t st);

// dst [n_rows, K] from src (and src2 for MAP_DUAL) in the tensor-core row order.
cudaError_t tc_rows_permute(int map, int8_t* dst, const int8_t* src, const int8_t* src2, int n_rows, int K,
                            cudaStream_t st);

#ifdef DEC_PROJ_TC_DEFINE

#ifdef DEC_PROJ_TC_PERMUTE_DEFINE
template <int MAP>
__global__ void k_tc_rows_permute(int8_t* __restrict__ dst, const int8_t* __restrict__ src,
                                  const int8_t* __restrict__ src2, int n_rows, int K) {
    const int p = blockIdx.x;
    if (p >= n_rows) return;
    const int n = tc_logical_row<MAP>(p);
    const int8_t* s = (MAP == MAP_DUAL && (p & 1)) ? src2 : src;
    const uint4* from = reinterpret_cast<const uint4*>(s + static_cast<long long>(n) * K);
    uint4* to = reinterpret_cast<uint4*>(dst + static_cast<long long>(p) * K);
    for (int k = threadIdx.x; k < K / 16; k += blockDim.x) to[k] = from[k];
}

cudaError_t tc_rows_permute(int map, int8_t* dst, const int8_t* src, const int8_t* src2, int n_rows, int K,
                            cudaStream_t st) {
    if (K % 16 != 0 || n_rows <= 0) return cudaErrorInvalidValue;
    if (map == MAP_ROPE) {
        if (n_rows % 64 != 0) return cudaErrorInvalidValue;
        k_tc_rows_permute<MAP_ROPE><<<n_rows, 128, 0, st>>>(dst, src, src2, n_rows, K);
    } else if (map == MAP_DUAL) {
        if (n_rows % 2 != 0) return cudaErrorInvalidValue;
        k_tc_rows_permute<MAP_DUAL><<<n_rows, 128, 0, st>>>(dst, src, src2, n_rows, K);
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}
#endif  // DEC_PROJ_TC_PERMUTE_DEFINE

template <int BT, int EPI, int MAP, int XD, int WD>
cudaError_t proj_tc_launch_bt(int num_sms, TcArgs A, int n_blocks, cudaStream_t st) {
    auto kern = k_proj_tc<BT, EPI, MAP, XD, WD>;
    constexpr int kStage = WD * kTcStageBytes;
    const int nch = (A.ksl + kTcKC - 1) / kTcKC;
    const size_t xbytes = size_t(XD) * nch * BT * 128;
    const size_t avail = size_t(227 * 1024) - 1024 - 1024 - xbytes;
    const int ns_max = int(std::min<size_t>(kTcMaxStages, avail / kStage));
    if (ns_max < 2) return cudaErrorNotSupported;
    thread_local int attr_dev = -1;   // attributes are per device; set again when it changes
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (attr_dev != dev) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024 - 1024);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        attr_dev = dev;
    }
    const int gy = (A.g.B + BT - 1) / BT;
    A.n_by = gy;
    // one CTA per SM (TMEM and the ring); the ring holds no more stages than a CTA streams
    const int cps = std::max(1, std::min(n_blocks, std::max(1, num_sms / gy) / A.n_ks));
    const int NS = std::min(ns_max, std::max(2, ((n_blocks + cps - 1) / cps) * nch));
    const size_t smem = 1024 + size_t(NS) * kStage + xbytes;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cps * A.n_ks * gy);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, A, NS);
}

template <int EPI, int MAP, int XD, int WD>
cudaError_t proj_tc_launch(int num_sms, const CUtensorMap& wmap, const CUtensorMap& xmap16, const CUtensorMap& xmap32,
                           int n_rows, int MB, const float* xs, void* part, size_t part_bytes, int* cnt, int cnt_len,
                           const GemvArgs& g, cudaStream_t st) {
    if (g.B < 1 || g.B > MB) return cudaErrorNotSupported;
    const MmaPlan p = tc_plan(n_rows, g.K, num_sms, XD);
    if (!p.ok) return cudaErrorNotSupported;
    if (p.n_ks > 1 && (tc_part_bytes(p, g.B, XD) > part_bytes || tc_counters(p, g.B) > cnt_len))
        return cudaErrorNotSupported;
    TcArgs A;
    A.wmap = wmap;
    A.xs = xs;
    A.part = static_cast<int*>(part);
    A.cnt = cnt;
    A.n_ks = p.n_ks;
    A.ksl = p.ksl;
    A.n_rows = n_rows;
    A.n_by = 1;
    A.MB = MB;
    A.g = g;
    if (g.B <= 16) {
        A.xmap = xmap16;
        return proj_tc_launch_bt<16, EPI, MAP, XD, WD>(num_sms, A, p.n_blocks, st);
    }
    A.xmap = xmap32;
    return proj_tc_launch_bt<32, EPI, MAP, XD, WD>(num_sms, A, p.n_blocks, st);
}

#define DEC_PROJ_TC_INSTANTIATE(EPI, MAP, XD, WD)                                                                 \
    template cudaError_t proj_tc_launch<EPI, MAP, XD, WD>(int, const CUtensorMap&, const CUtensorMap&,           \
                                                          const CUtensorMap&, int, int, const float*, void*, size_t, \
                                                          int*, int, const GemvArgs&, cudaStream_t);

#endif  // DEC_PROJ_TC_DEFINE

}  // namespace dec
