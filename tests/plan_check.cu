// Host-only checks of the tensor-core launch plans (no GPU needed): for every projection
// shape of the workloads and test models and every batch size, the K split covers K
// exactly, slices are whole pipeline stages, the staged activation slice fits its budget,
// the split-K scratch and counters hold every index the kernels write, the plan does not
// depend on the batch, and the tensor-core head's shared memory fits. Prints one line per
// failure and "ok" at the end; exits non-zero on any failure.
#include <cstdio>
#include <vector>

#include "dec.h"
#include "chain_plan.h"
#include "head_tc.cuh"
#include "proj_mma.cuh"
#include "proj_tc.cuh"

using namespace dec;

static int failures = 0;
#define CHECK(cond, ...)                   \
    do {                                   \
        if (!(cond)) {                     \
            ++failures;                    \
            std::printf("FAIL: " __VA_ARGS__); \
            std::printf("\n");             \
        }                                  \
    } while (0)

struct Shape {
    int N, K, elt;   // elt 4: f32 weights, 1: int8 weights (TF32 kernel); 0: W8A8 (tcgen05)
};

int main() {
    const int sms = 148;
    // chains of a split step: cover the batch exactly, at least kMmaMinBatch rows each,
    // at most kMaxChains, in ascending order
    for (int B = 1; B <= DEC_MAX_BATCH; ++B) {
        int r0[kMaxChains + 1];
        const int n = chain_bounds(B, r0);
        CHECK(n >= 1 && n <= kMaxChains, "chain count B=%d n=%d", B, n);
        CHECK(r0[0] == 0 && r0[n] == B, "chains cover B=%d", B);
        for (int c = 0; c < n; ++c) {
            CHECK(r0[c + 1] > r0[c], "chain order B=%d", B);
            if (B >= kSplitMinBatch) CHECK(r0[c + 1] - r0[c] >= kMmaMinBatch, "chain rows B=%d c=%d", B, c);
        }
        if (B >= kSplitMinBatch) CHECK(n == kMaxChains, "split B=%d n=%d", B, n);
        std::printf("chain %d %d %d\n", B, n, r0[1]);
    }
    // (d, F, V, family W8A8?, f32?)
    struct Model {
        int d, F, V;
        int kind;   // 0 f32 whisper, 1 W8A32 whisper, 2 W8A8 qwen2
        int kvd;    // K/V width (grouped-query attention); 0: d
    } models[] = {{384, 1536, 51865, 0, 0},  {512, 2048, 51865, 0, 0}, {1024, 2816, 151936, 2, 0},
                  {1280, 5120, 51866, 1, 0}, {128, 384, 1031, 0, 0},   {192, 320, 997, 1, 0},
                  {128, 352, 1009, 2, 0},    {256, 704, 4099, 2, 0},   {256, 2048, 1031, 0, 0},
                  {896, 2432, 1009, 2, 0},   {256, 352, 1009, 2, 128}, {896, 2432, 1009, 2, 128},
                  {896, 4864, 151936, 2, 128}};
    for (const auto& m : models) {
        std::vector<Shape> shapes;
        const int d = m.d, F = m.F, kvd = m.kvd ? m.kvd : m.d;
        if (m.kind == 2) {
            shapes = {{d + 2 * kvd, d, 0}, {d, d, 0}, {2 * F, d, 0}, {d, F, 0}};
        } else {
            const int e = m.kind == 0 ? 4 : 1;
            shapes = {{3 * d, d, e}, {d, d, e}, {F, d, e}, {d, F, e}};
        }
        shapes.push_back({m.V, d, 4});   // f32 head on the TF32 kernel (fallback path)
        // Whisper projections on the tcgen05 digit path (three activation planes)
        if (m.kind != 2) {
            for (const auto& s : shapes) {
                if (s.N == m.V) continue;
                const MmaPlan p = tc_plan(s.N, s.K, sms, 3);
                CHECK(p.ok, "digit plan not ok N=%d K=%d", s.N, s.K);
                if (!p.ok) continue;
                CHECK(p.n_ks * p.ksl >= s.K && (p.n_ks - 1) * p.ksl < s.K, "digit K cover N=%d K=%d", s.N, s.K);
                CHECK(p.ksl % kTcKC == 0 || p.ksl == s.K, "digit slice not whole stages N=%d K=%d", s.N, s.K);
                const int nch = (p.ksl + kTcKC - 1) / kTcKC;
                CHECK(size_t(3) * kTcMaxBT * nch * 128 <= kTcXBudget, "digit X budget N=%d K=%d", s.N, s.K);
                for (int wd : {1, 3}) {
                    // ring: at least two stages of wd weight planes next to the activation slice
                    const size_t avail = size_t(227 * 1024) - 2048 - size_t(3) * nch * kTcMaxBT * 128;
                    CHECK(avail / (size_t(wd) * kTcStageBytes) >= 2, "digit ring N=%d K=%d wd=%d", s.N, s.K, wd);
                }
                for (int B = 1; B <= DEC_MAX_BATCH; ++B) {
                    const int BT = B <= 16 ? 16 : 32;
                    const int gy = (B + BT - 1) / BT;
                    // part[((grp * n_ks + ks) * 32 + lane) * 3 * (BT / 2) + v], grp < n_blocks * gy * 8
                    const size_t need = size_t(p.n_blocks) * gy * 8 * p.n_ks * 32 * 3 * (BT / 2) * 4;
                    if (p.n_ks > 1) CHECK(need <= tc_part_bytes(p, B, 3), "digit scratch N=%d K=%d B=%d", s.N, s.K, B);
                    CHECK(p.n_blocks * gy * 8 <= tc_counters(p, B), "digit counters N=%d K=%d B=%d", s.N, s.K, B);
                    for (int sets = 1; sets <= 2; ++sets)
                        CHECK(tc_tmem_cols(3, BT, sets) <= 256 && uint32_t(sets * 3 * BT) <= tc_tmem_cols(3, BT, sets),
                              "digit TMEM columns B=%d", B);
                    // stacked planes: MMA N = 3 BT, 2 BT, BT within the M = 128 limits
                    CHECK(3 * BT <= 256 && (3 * BT) % 16 == 0 && (2 * BT) % 16 == 0 && BT % 16 == 0,
                          "digit MMA N B=%d", B);
                }
            }
        }
        for (int bt : {16, 32})
            for (int sets = 1; sets <= 2; ++sets)
                CHECK(tc_tmem_cols(1, bt, sets) <= 256 && uint32_t(sets * bt) <= tc_tmem_cols(1, bt, sets),
                      "W8A8 TMEM columns");
        for (const auto& s : shapes) {
            if (s.elt == 0) {
                const MmaPlan p = tc_plan(s.N, s.K, sms);
                CHECK(p.ok, "tc_plan not ok N=%d K=%d", s.N, s.K);
                if (!p.ok) continue;
                CHECK(p.n_ks * p.ksl >= s.K && (p.n_ks - 1) * p.ksl < s.K, "tc K cover N=%d K=%d", s.N, s.K);
                CHECK(p.ksl % kTcKC == 0 || p.ksl == s.K, "tc slice not whole stages N=%d K=%d", s.N, s.K);
                const int nch = (p.ksl + kTcKC - 1) / kTcKC;
                CHECK(size_t(kTcMaxBT) * nch * 128 <= kTcXBudget, "tc X budget N=%d K=%d", s.N, s.K);
                for (int B = 1; B <= DEC_MAX_BATCH; ++B) {
                    const int BT = B <= 16 ? 16 : 32;
                    const int gy = (B + BT - 1) / BT;
                    // kernel: part[((grp * n_ks + ks) * 32 + lane) * (BT / 2) + col],
                    // grp < n_blocks * gy * 4 lane quarters * 2 column halves
                    const size_t need = size_t(p.n_blocks) * gy * 4 * 2 * p.n_ks * 32 * (BT / 2) * 4;
                    if (p.n_ks > 1) CHECK(need <= tc_part_bytes(p, B), "tc scratch N=%d K=%d B=%d", s.N, s.K, B);
                    CHECK(p.n_blocks * gy * 4 * 2 <= tc_counters(p, B), "tc counters N=%d K=%d B=%d", s.N, s.K, B);
                    const MmaPlan q = tc_plan(s.N, s.K, sms);
                    CHECK(q.n_ks == p.n_ks && q.ksl == p.ksl, "tc plan depends on call");
                }
            } else {
                const MmaPlan p = mma_plan(s.N, s.K, s.elt, sms);
                if (!p.ok) continue;   // the CUDA-core kernel runs instead
                const int KC = p.nbx * 128 / s.elt;
                CHECK(p.n_ks * p.ksl >= s.K && (p.n_ks - 1) * p.ksl < s.K, "mma K cover N=%d K=%d", s.N, s.K);
                CHECK(p.ksl % KC == 0 || p.ksl == s.K, "mma slice not whole stages N=%d K=%d", s.N, s.K);
                CHECK(p.ksl % 32 == 0, "mma slice not a multiple of 32 N=%d K=%d", s.N, s.K);
                const int pad = s.elt == 4 ? 4 : 16;
                CHECK(size_t(kMmaMaxBT) * (p.ksl + pad) * 4 <= kMmaXBudget, "mma X budget N=%d K=%d", s.N, s.K);
                for (int B = 8; B <= DEC_MAX_BATCH; ++B) {
                    int BT = 8;
                    while (BT < B && BT < kMmaMaxBT) BT <<= 1;
                    const int gy = (B + BT - 1) / BT;
                    // kernel: tile ((jb * n_by + by) * n_ks + ks) * 128 * BT floats
                    const size_t need = size_t(p.n_blocks) * gy * p.n_ks * 128 * BT * 4;
                    if (p.n_ks > 1) CHECK(need <= mma_part_bytes(p, B), "mma scratch N=%d K=%d B=%d", s.N, s.K, B);
                    CHECK(p.n_blocks * gy * kMmaConsumerWarps <= mma_counters(p, B), "mma counters N=%d K=%d B=%d",
                          s.N, s.K, B);
                }
            }
        }
        // the tensor-core head: hidden planes plus at least two weight stages fit
        for (int bt : {16, 32}) {
            const int ns = head_tc_stages(d, bt);
            CHECK(ns >= 2, "head stages d=%d bt=%d", d, bt);
            CHECK(head_tc_smem(d, bt, ns) <= size_t(227 * 1024 - 1024), "head smem d=%d bt=%d", d, bt);
        }
    }
    // digit sums stay inside int32 for every K the head accepts
    CHECK(3LL * 127 * 127 * kHeadMaxK < (1LL << 31), "int32 head sums");
    std::printf(failures ? "%d failures\n" : "ok\n", failures);
    return failures ? 1 : 0;
}
