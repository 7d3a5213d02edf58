// C ABI of the batched single-token decoder step (see include/dec.h).
//
// Host side: validation before any launch, weight packing at create time, one
// launch sequence per step on the caller's stream (programmatic dependent launch
// between kernels), and the handle's bookkeeping of slot lengths.

#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <type_traits>
#include <array>
#include <map>
#include <vector>

#include "../../include/dec.h"
#include "attention.cuh"
#include "attn_plan.h"
#include "chain_plan.h"
#include "common.cuh"
#include "gemv.cuh"
#include "gemv_launch.cuh"
#include "misc.cuh"
#include "head_tc.cuh"
#include "rowprep_i8.cuh"
#include "proj_tc.cuh"
#include "proj_mma.cuh"

using namespace dec;

namespace {

constexpr int kMetaRing = 8;
// Prompt tokens of one slot that dec_prefill runs together as one step's rows.
constexpr int kPrefillChunk = DEC_MAX_BATCH;
constexpr int kMaxSplits = kAttnMaxSplits;

thread_local std::string g_create_error;
// Allocation-failure injection for tests (dec_debug_fail_alloc): the n-th allocation of the
// next dec_create on this thread fails; 0 disables.
thread_local int g_fail_alloc_at = 0;
thread_local int g_alloc_count = 0;

}  // namespace

// Message for dec_last_error(NULL) from handle-less entry points in other files.
void dec_set_thread_error(const char* msg) { g_create_error = msg ? msg : ""; }

namespace {

struct LayerDev {
    float *n1w = nullptr, *n1b = nullptr, *n2w = nullptr, *n2b = nullptr, *n3w = nullptr, *n3b = nullptr;
    void* wqkv = nullptr;
    float *sqkv = nullptr, *bqkv = nullptr;
    void* wo = nullptr;
    float *so = nullptr, *bo = nullptr;
    void *wxq = nullptr, *wxk = nullptr, *wxv = nullptr, *wxo = nullptr;
    float *sxq = nullptr, *sxk = nullptr, *sxv = nullptr, *sxo = nullptr;
    float *bxq = nullptr, *bxk = nullptr, *bxv = nullptr, *bxo = nullptr;
    void *w1 = nullptr, *w2 = nullptr;
    float *s1 = nullptr, *s2 = nullptr, *b1 = nullptr, *b2 = nullptr;
    void *wg = nullptr, *wu = nullptr, *wd = nullptr;
    float *sg = nullptr, *su = nullptr, *sd = nullptr;
    // Qwen tensor-core path: q|k|v rows in RoPE pair order, gate/up rows interleaved
    void *wqkv_p = nullptr, *wgu = nullptr;
    // 2-D TMA descriptors of the projections (tensor-core path); Qwen uses m_qkv (the
    // permuted panel), m_o, m_1 (gate/up) and m_2 (down)
    CUtensorMap m_qkv, m_o, m_xq, m_xo, m_1, m_2;
};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

}  // namespace

// Per-chain step scratch. A decode step of many rows runs as up to kMaxChains chains over
// equal parts of the rows, on their own streams, so that the chains' latency-bound kernels
// overlap one another and the attention of one. Each chain has its own copies of everything
// a launch writes besides its rows of x, so chains never share scratch.
struct Chain {
    float *q = nullptr, *ctx = nullptr, *ffn = nullptr, *xq = nullptr;
    float* part = nullptr;          // attention split partials
    int* counters = nullptr;        // attention split arrival counts, zero between launches
    float* xn = nullptr;            // normalised activation rows (TF32 tensor-core path)
    int8_t* xq8 = nullptr;          // quantised activation rows and their scales (int8 tensor-core path)
    int xq8_rows = 0;               // rows of xq8 (>= max batch, >= 32)
    CUtensorMap m_xq8[2][2];        // xq8 as [rows, K] for K = d, F and boxes of 16, 32 rows
    float* xs8 = nullptr;
    // Whisper tcgen05 path: activation rows as three int8 digit planes [3][xd_rows][K]
    int8_t* xd3 = nullptr;
    float* xsd = nullptr;
    int xd_rows = 0;
    CUtensorMap m_xd3[2][2];        // xd3 as [3 rows, K] for K = d, F and boxes of 16, 32 rows
    void* mma_part = nullptr;       // split-K partial tiles (tensor-core path)
    size_t mma_part_bytes = 0;
    int* mma_cnt = nullptr;         // split-K arrival counts, zero between launches
    int mma_cnt_len = 0;
    StepMeta* meta = nullptr;       // the chain's rows of the step description
};

struct dec_handle {
    dec_config cfg{};
    int device = 0;
    int num_sms = 148;
    std::vector<void*> dallocs;
    std::vector<void*> hallocs;
    float *tok_emb = nullptr, *pos_emb = nullptr, *final_w = nullptr, *final_b = nullptr;
    float2* rope = nullptr;
    CUtensorMap m_head;            // TMA descriptor of the tied head (tensor-core path)
    bool tma_ok = false;           // descriptors built (else the CUDA-core path is used)
    // tcgen05 head: embedding and hidden rows as three int8 digit planes with row scales
    int8_t *wdig = nullptr, *xdig = nullptr;
    float *wsc = nullptr, *xsc = nullptr;
    int* xsum = nullptr;            // per hidden row: sum |D1|, sum |D2| (int8 head bound)
    float* head_thr = nullptr;      // int8 head: per-row candidate threshold
    int* head_cand = nullptr;       // int8 head: candidate list (max_batch * vocab)
    float* head_logits = nullptr;   // int8 head: coarse logits when the caller passes none
    int xdig_rows = 0;             // rows per hidden digit plane (>= max batch, >= 32)
    CUtensorMap m_wdig, m_xdig16, m_xdig32;
    bool head_tc_ok = false;
    std::vector<LayerDev> layers;
    float *kc = nullptr, *vc = nullptr, *xkc = nullptr, *xvc = nullptr;
    // paged self-attention cache (page_rows > 0): a pool of pages shared by all slots and a
    // per-slot page table; a dense cache is one page of max_cache_len rows per slot
    int page_rows = 0, pages_per_slot = 1, n_pages = 0;
    int* d_table = nullptr;                    // [max_slots][pages_per_slot] physical pages
    std::vector<int> free_pages;
    std::vector<std::vector<int>> slot_pages;
    long long self_slot_stride = 0, self_layer_stride = 0, cross_slot_stride = 0, cross_layer_stride = 0;
    int max_batch = 0;
    int max_rows = 0;                  // rows of the per-step workspaces: max(max_batch, prompt chunk)
    int prefill_chunk = kPrefillChunk; // prompt rows per prefill step
    int tps_self = 1, tps_cross = 1;   // attention tiles per split (handle constants)
    // workspace: the residual rows x are shared by both chains (each owns a row range); the
    // rest of the per-step scratch is per chain (see Chain)
    float* x = nullptr;
    Chain chain[kMaxChains];
    Chain* w = &chain[0];           // the chain whose launches are being issued
    int n_chains = 1;               // chains allocated: up to kMaxChains when batches can be split
    cudaStream_t side = nullptr;    // the second chain's stream (eager steps)
    cudaStream_t side_streams[kMaxChains] = {};   // chain c > 0 runs on side_streams[c] (eager steps)
    cudaEvent_t ev_fork = nullptr, ev_join[kMaxChains] = {};
    bool tcd_ok = false;            // Whisper digit-path descriptors and planes built
    unsigned long long* keys = nullptr;
    int* head_counter = nullptr;
    int* last_tok = nullptr;
    int* dev_err = nullptr;
    int* host_status = nullptr;     // pinned copy of the status word after dec_step_host
    int* host_tok = nullptr;        // pinned copy of every slot's greedy continuation token
    bool failed = false;            // a bounded device wait gave up; dec_reset required
    int inject_drop = 0;            // test hook: drop one attention tile copy per step
    StepMeta* dmeta = nullptr;      // [3]: the whole step, then the rows of chain 0 and chain 1
    StepMeta* hmeta[kMetaRing] = {};
    cudaEvent_t hev[kMetaRing] = {};
    int ring = 0;
    // host view of the slots
    std::vector<int> slot_len;
    std::vector<char> has_tok, has_cross;
    int last_batch = 0;
    // CUDA graphs of the step's launch sequence, keyed by what changes its launches:
    // batch size, self-attention tile count, output pointers. A null entry means
    // capture failed for that key and the step runs eagerly.
    struct StepGraph {
        cudaGraphExec_t exec;
        int kernels;   // kernel launches in one step of this key (-1: not captured)
    };
    std::map<std::array<long long, 5>, StepGraph> graphs;
    float* trace = nullptr;          // per-layer residual copies [L, B, d], or null
    // per-phase device timing: an event after each phase of the most recent timed step
    bool phase_timing = false;
    std::vector<cudaEvent_t> phase_ev;
    std::vector<std::array<int, 2>> phase_tag;   // (layer, DEC_PHASE_*) of each event after the first
    size_t phase_n = 0;
    int last_step_kernels = -1;
    cudaStream_t cap_stream = nullptr;
    float* stage_logits = nullptr;   // dec_step_host result staging
    int* stage_argmax = nullptr;
    std::string err;
};

namespace {

dec_status fail(dec_handle* h, dec_status st, const std::string& msg) {
    if (h)
        h->err = msg;
    else
        g_create_error = msg;
    return st;
}

dec_status cuda_fail(dec_handle* h, cudaError_t e, const char* what) {
    return fail(h, DEC_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

#define DEC_CUDA(h, call)                                    \
    do {                                                     \
        cudaError_t e_ = (call);                             \
        if (e_ != cudaSuccess) return cuda_fail((h), e_, #call); \
    } while (0)

// The allocation-failure hook: true when this allocation is the one asked to fail.
bool injected_alloc_failure() { return g_fail_alloc_at > 0 && ++g_alloc_count == g_fail_alloc_at; }

template <typename T>
dec_status dalloc(dec_handle* h, T** p, size_t bytes) {
    void* q = nullptr;
    if (bytes == 0) bytes = 16;
    if (injected_alloc_failure())
        return fail(h, DEC_ENOMEM, "cudaMalloc of " + std::to_string(bytes) + " bytes failed (injected)");
    cudaError_t e = cudaMalloc(&q, bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(h, DEC_ENOMEM, "cudaMalloc of " + std::to_string(bytes) + " bytes failed");
    }
    h->dallocs.push_back(q);
    *p = static_cast<T*>(q);
    return DEC_OK;
}

template <typename T>
dec_status upload(dec_handle* h, T** dst, const void* src, size_t bytes) {
    dec_status st = dalloc(h, dst, bytes);
    if (st != DEC_OK) return st;
    DEC_CUDA(h, cudaMemcpy(*dst, src, bytes, cudaMemcpyHostToDevice));
    return DEC_OK;
}

#define DEC_TRY(x)                        \
    do {                                  \
        dec_status s_ = (x);              \
        if (s_ != DEC_OK) return s_;      \
    } while (0)

size_t wbytes(const dec_config& c) { return c.proj_fmt == DEC_PROJ_F32 ? 4 : 1; }
// K/V heads (grouped-query attention) and the K/V width
int kv_heads(const dec_config& c) { return c.n_kv_heads > 0 ? c.n_kv_heads : c.n_heads; }
int kv_width(const dec_config& c) { return kv_heads(c) * 64; }

// Where the self-attention cache rows live (see KvMap).
KvMap self_kv_map(const dec_handle* h);

// Upload a projection: weights [out, in], optional scales [out] and bias [out].
dec_status upload_proj(dec_handle* h, const dec_proj& p, int out, int in, bool want_bias, void** w, float** s,
                       float** b, const char* name) {
    const dec_config& c = h->cfg;
    if (!p.w) return fail(h, DEC_EINVAL, std::string("missing weights for ") + name);
    if (c.proj_fmt != DEC_PROJ_F32 && !p.scale) return fail(h, DEC_EINVAL, std::string("missing scales for ") + name);
    if (want_bias != (p.bias != nullptr))
        return fail(h, DEC_EINVAL, std::string(want_bias ? "missing bias for " : "unexpected bias for ") + name);
    DEC_TRY(upload(h, w, p.w, size_t(out) * in * wbytes(c)));
    if (c.proj_fmt != DEC_PROJ_F32) DEC_TRY(upload(h, s, p.scale, size_t(out) * 4));
    if (p.bias) DEC_TRY(upload(h, b, p.bias, size_t(out) * 4));
    return DEC_OK;
}

// Fused q|k|v panel [3d, d] with its scales and biases (franken_ocr decoder_qwen2.rs, `concat_qkv`).
dec_status upload_qkv(dec_handle* h, const dec_layer_weights& L, LayerDev& D) {
    const dec_config& c = h->cfg;
    const int d = c.d_model, kvd = kv_width(c);
    const size_t wb = wbytes(c);
    const dec_proj* ps[3] = {&L.q, &L.k, &L.v};
    const int rows[3] = {d, kvd, kvd};        // q [d, d], k and v [kv width, d]
    const int off[3] = {0, d, d + kvd};       // first row of each section in the panel
    for (int i = 0; i < 3; ++i) {
        if (!ps[i]->w) return fail(h, DEC_EINVAL, "missing q/k/v weights");
        if (c.proj_fmt != DEC_PROJ_F32 && !ps[i]->scale) return fail(h, DEC_EINVAL, "missing q/k/v scales");
        if (!ps[i]->bias) return fail(h, DEC_EINVAL, "missing q/k/v bias");
    }
    const int n_rows = d + 2 * kvd;
    DEC_TRY(dalloc(h, &D.wqkv, size_t(n_rows) * d * wb));
    DEC_TRY(dalloc(h, &D.bqkv, size_t(n_rows) * 4));
    if (c.proj_fmt != DEC_PROJ_F32) DEC_TRY(dalloc(h, &D.sqkv, size_t(n_rows) * 4));
    for (int i = 0; i < 3; ++i) {
        DEC_CUDA(h, cudaMemcpy(static_cast<char*>(D.wqkv) + size_t(off[i]) * d * wb, ps[i]->w,
                               size_t(rows[i]) * d * wb, cudaMemcpyHostToDevice));
        DEC_CUDA(h, cudaMemcpy(D.bqkv + off[i], ps[i]->bias, size_t(rows[i]) * 4, cudaMemcpyHostToDevice));
        if (D.sqkv)
            DEC_CUDA(h, cudaMemcpy(D.sqkv + off[i], ps[i]->scale, size_t(rows[i]) * 4, cudaMemcpyHostToDevice));
    }
    return DEC_OK;
}

dec_status validate_config(const dec_config& c) {
    auto bad = [](const std::string& m) { return fail(nullptr, DEC_EINVAL, m); };
    if (c.family != DEC_FAMILY_WHISPER && c.family != DEC_FAMILY_QWEN2) return bad("unknown family");
    if (c.head_dim != 64) return bad("head_dim must be 64");
    if (c.n_heads < 1 || c.d_model != c.n_heads * 64) return bad("d_model must equal n_heads * 64");
    if (c.n_kv_heads < 0 || (c.n_kv_heads > 0 && c.n_heads % c.n_kv_heads != 0))
        return bad("n_kv_heads must divide n_heads (0: one K/V head per query head)");
    if (c.family == DEC_FAMILY_WHISPER && c.n_kv_heads > 0 && c.n_kv_heads != c.n_heads)
        return bad("grouped-query attention is a qwen2 option");
    if (c.n_layers < 1) return bad("n_layers must be >= 1");
    if (c.d_ff < 16 || c.d_ff % 16) return bad("d_ff must be a positive multiple of 16");
    if (c.vocab < 1) return bad("vocab must be >= 1");
    if (c.max_pos < 1) return bad("max_pos must be >= 1");
    if (c.max_slots < 1) return bad("max_slots must be >= 1");
    if (c.max_cache_len < 1) return bad("max_cache_len must be >= 1");
    if (!(c.norm_eps > 0.0f)) return bad("norm_eps must be > 0");
    if (c.head_fmt != DEC_HEAD_EXACT && c.head_fmt != DEC_HEAD_INT8_REFINE) return bad("unknown head_fmt");
    if (c.kv_page_rows != 0 && c.kv_page_rows != 16 && c.kv_page_rows != 32 && c.kv_page_rows != 64)
        return bad("kv_page_rows must be 0 (dense), 16, 32 or 64");
    if (c.kv_page_rows > 0 && c.kv_pages < 1) return bad("a paged cache needs kv_pages >= 1");
    if (c.head_fmt == DEC_HEAD_INT8_REFINE &&
        (c.d_model > 4096 || static_cast<long long>(c.vocab) * DEC_MAX_BATCH >= (1LL << 31)))
        return bad("the int8 head needs d_model <= 4096 and vocab * 128 < 2^31");
    if (c.family == DEC_FAMILY_WHISPER) {
        if (c.enc_len < 1) return bad("whisper needs enc_len >= 1");
        if (c.proj_fmt != DEC_PROJ_F32 && c.proj_fmt != DEC_PROJ_W8A32)
            return bad("whisper supports f32 or w8a32 projections");
    } else {
        if (c.proj_fmt != DEC_PROJ_W8A8) return bad("qwen2 supports w8a8 projections");
        if (!(c.rope_theta > 0.0f)) return bad("rope_theta must be > 0");
        if (c.max_pos > (1 << 22)) return bad("max_pos too large for the RoPE table");
    }
    return DEC_OK;
}

// NEOX RoPE table: angle = pos * theta^(-2i/64) in double, cos and sin rounded to f32.
dec_status build_rope(dec_handle* h) {
    const dec_config& c = h->cfg;
    std::vector<float2> t(size_t(c.max_pos) * 32);
    for (int p = 0; p < c.max_pos; ++p)
        for (int i = 0; i < 32; ++i) {
            const double inv = std::pow(double(c.rope_theta), -2.0 * i / 64.0);
            const double ang = double(p) * inv;
            t[size_t(p) * 32 + i] = make_float2(float(std::cos(ang)), float(std::sin(ang)));
        }
    return upload(h, &h->rope, t.data(), t.size() * sizeof(float2));
}

// ------------------------------------------------------------------ launches

template <typename K, typename... Args>
cudaError_t launch(K kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}


template <typename WT, bool I8, int PRO, int EPI, int MAP>
dec_status gemv(dec_handle* h, const GemvArgs& a, cudaStream_t st) {
    cudaError_t e = gemv_launch<WT, I8, PRO, EPI, MAP>(h->num_sms, a, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "projection kernel launch");
    return DEC_OK;
}

// Batches of at least kMmaMinBatch rows (chain_plan.h) can take the tensor-core projection
// paths. Which path runs also depends on the matrix (measured per shape on B200, PDL chains
// with weights streamed from HBM): below about 2^21 weights with K < 2048 the tensor-core
// kernels' fixed cost (activation slice load, split-K exchange) is larger than the
// CUDA-core kernel's whole run, except for int8 weights with f32 activations, whose
// CUDA-core kernel is arithmetic-bound from batch 8 on.
constexpr long long kMmaMinWeights = 1LL << 21;

bool mma_worth(int N, int K, bool w8a32) {
    return w8a32 || K >= 2048 || static_cast<long long>(N) * K >= 4 * kMmaMinWeights;
}

bool mma_eligible(const dec_handle* h, int N, int K, int elt, int B) {
    if (!h->tma_ok || B < kMmaMinBatch) return false;
    const MmaPlan p = mma_plan(N, K, elt, h->num_sms);
    if (!p.ok || K > kRowprepMaxK) return false;
    return p.n_ks == 1 || (mma_part_bytes(p, B) <= h->w->mma_part_bytes && mma_counters(p, B) <= h->w->mma_cnt_len);
}

// Norm prologue of the tensor-core path: normalised rows into h->w->xn, which becomes the
// projection's input.
template <int PRO>
dec_status mma_input(dec_handle* h, GemvArgs& g, cudaStream_t st) {
    if (PRO == PRO_NONE) return DEC_OK;
    const cudaError_t e = rowprep_launch<PRO>(g, h->w->xn, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "row normalisation launch");
    g.x = h->w->xn;
    g.x_ld = g.K;
    return DEC_OK;
}

template <typename WT, int PRO, int EPI>
dec_status proj_mma(dec_handle* h, const GemvArgs& a, const CUtensorMap& map, cudaStream_t st) {
    GemvArgs g = a;
    DEC_TRY(mma_input<PRO>(h, g, st));
    const cudaError_t e =
        proj_mma_launch<WT, EPI>(h->num_sms, map, h->w->mma_part, h->w->mma_part_bytes, h->w->mma_cnt, h->w->mma_cnt_len, g, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "tensor-core projection launch");
    return DEC_OK;
}

bool tc_eligible(const dec_handle* h, int n_rows, int K, int B) {
    if (!h->tma_ok || B < kMmaMinBatch) return false;
    const MmaPlan p = tc_plan(n_rows, K, h->num_sms);
    if (!p.ok) return false;
    return p.n_ks == 1 || (tc_part_bytes(p, B) <= h->w->mma_part_bytes && tc_counters(p, B) <= h->w->mma_cnt_len);
}

// W8A8 on tcgen05 int8 tensor cores: rows quantised by k_rowprep_i8, exact int32 products.
template <int PRO, int EPI, int MAP>
dec_status proj_w8a8_tc(dec_handle* h, const GemvArgs& a, const CUtensorMap& map, int n_rows, cudaStream_t st) {
    cudaError_t e = rowprep_i8_launch<PRO>(a, h->w->xq8, h->w->xs8, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "row quantisation launch");
    const int kx = a.K == h->cfg.d_model ? 0 : 1;
    e = proj_tc_launch<EPI, MAP, 1, 1>(h->num_sms, map, h->w->m_xq8[kx][0], h->w->m_xq8[kx][1], n_rows, h->w->xq8_rows, h->w->xs8,
                                       h->w->mma_part, h->w->mma_part_bytes, h->w->mma_cnt, h->w->mma_cnt_len, a, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "tcgen05 projection launch");
    return DEC_OK;
}

bool tcd_eligible(const dec_handle* h, int N, int K, int B) {
    if (!h->tcd_ok || B < kMmaMinBatch || B > h->w->xd_rows) return false;
    const MmaPlan p = tc_plan(N, K, h->num_sms, 3);
    if (!p.ok) return false;
    return p.n_ks == 1 || (tc_part_bytes(p, B, 3) <= h->w->mma_part_bytes && tc_counters(p, B) <= h->w->mma_cnt_len);
}

// Whisper projections on tcgen05 int8 tensor cores: the (normalised) activation rows split
// into three int8 digit planes by k_rowprep_digits, times the int8 weights (W8A32, one
// plane, three products per K step) or the f32 weights' three digit planes (six products),
// with exact int32 sums; y = s_n s_b (A0 + (A1 + A2 / 254) / 254) + bias.
template <int PRO, int EPI>
dec_status proj_digits_tc(dec_handle* h, const GemvArgs& a, const LayerDev* L, int m, cudaStream_t st) {
    cudaError_t e = rowprep_digits_launch<PRO>(a.x, a.x_ld, a.norm_w, a.norm_b, a.eps, a.K, a.B,
                                               static_cast<long long>(h->w->xd_rows) * a.K, h->w->xd3, h->w->xsd,
                                               nullptr, true, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "row digit split launch");
    const int kx = a.K == h->cfg.d_model ? 0 : 1;
    const CUtensorMap* maps[6] = {&L->m_qkv, &L->m_o, &L->m_xq, &L->m_xo, &L->m_1, &L->m_2};
    e = proj_tc_launch<EPI, MAP_ADJ, 3, 1>(h->num_sms, *maps[m], h->w->m_xd3[kx][0], h->w->m_xd3[kx][1], a.N,
                                           h->w->xd_rows, h->w->xsd, h->w->mma_part, h->w->mma_part_bytes,
                                           h->w->mma_cnt, h->w->mma_cnt_len, a, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "tcgen05 digit projection launch");
    return DEC_OK;
}

// Whisper projections exist as f32 or W8A32: from batch 8 on, tcgen05 on digit planes (or
// TF32 mma.sync when those are unavailable), the CUDA-core kernel below. `m` names the
// layer's matrix (0 q|k|v, 1 o, 2 cross q, 3 cross o, 4 fc1, 5 fc2).
template <int PRO, int EPI, int MAP>
dec_status gemv_whisper(dec_handle* h, const GemvArgs& a, cudaStream_t st, const LayerDev& layer, int m) {
    const bool f32w = h->cfg.proj_fmt == DEC_PROJ_F32;
    const LayerDev* L = &layer;
    if (h->tma_ok) {
        // W8A32 on the digit path; f32 weights stay on TF32 / CUDA cores (a three-plane digit
        // path for them measured slower at the C2 shapes: its row split is a launch of its
        // own and fc2's activation planes need a split-K exchange)
        if (!f32w && tcd_eligible(h, a.N, a.K, a.B)) return proj_digits_tc<PRO, EPI>(h, a, L, m, st);
        const CUtensorMap* maps[6] = {&L->m_qkv, &L->m_o, &L->m_xq, &L->m_xo, &L->m_1, &L->m_2};
        if (f32w && mma_worth(a.N, a.K, false) && mma_eligible(h, a.N, a.K, 4, a.B))
            return proj_mma<float, PRO, EPI>(h, a, *maps[m], st);
        if (!f32w && mma_eligible(h, a.N, a.K, 1, a.B)) return proj_mma<int8_t, PRO, EPI>(h, a, *maps[m], st);
    }
    if (f32w) return gemv<float, false, PRO, EPI, MAP>(h, a, st);
    return gemv<int8_t, false, PRO, EPI, MAP>(h, a, st);
}

// Qwen W8A8 projections: tcgen05 int8 tensor cores from batch 8 on, dp4a below
// (bit-identical: exact int32 sums from the same int8 codes).
template <int PRO, int EPI, int MAP>
dec_status gemv_qwen(dec_handle* h, const GemvArgs& a, const CUtensorMap& map, cudaStream_t st) {
    const int n_rows = MAP == MAP_DUAL ? 2 * a.N : a.N;
    if (tc_eligible(h, n_rows, a.K, a.B)) return proj_w8a8_tc<PRO, EPI, MAP>(h, a, map, n_rows, st);
    return gemv<int8_t, true, PRO, EPI, MAP>(h, a, st);
}

// Final norm + tied head with the greedy argmax: tcgen05 int8 tensor cores on digit
// planes at every batch size when they were built, else TF32 tensor cores from batch 8
// on and CUDA cores below.
template <int PRO>
dec_status head(dec_handle* h, const GemvArgs& a, cudaStream_t st) {
    if (h->head_tc_ok) {
        const int d = h->cfg.d_model;
        const bool int8_head = h->cfg.head_fmt == DEC_HEAD_INT8_REFINE;
        // batches above 16 (and the int8 head, whose refine kernel reads them): the hidden
        // rows' digit planes come from their own kernel; smaller batches of the exact head make
        // them inside the head kernel (same arithmetic)
        const bool own = !int8_head && head_tc_makes_planes(a.B);
        cudaError_t e = cudaSuccess;
        if (!own) {
            e = rowprep_digits_launch<PRO>(a.x, a.x_ld, a.norm_w, a.norm_b, a.eps, d, a.B,
                                           static_cast<long long>(h->xdig_rows) * d, h->xdig, h->xsc, h->xsum, true,
                                           st);
            if (e != cudaSuccess) return cuda_fail(h, e, "head row split launch");
        }
        HeadArgs ha;
        ha.wmap = h->m_wdig;
        ha.xmap16 = h->m_xdig16;
        ha.xmap32 = h->m_xdig32;
        ha.wscale = h->wsc;
        ha.xscale = h->xsc;
        ha.x = a.x;
        ha.x_ld = a.x_ld;
        ha.norm_w = a.norm_w;
        ha.norm_b = a.norm_b;
        ha.eps = a.eps;
        ha.V = h->cfg.vocab;
        ha.K = d;
        ha.B = a.B;
        ha.MB = h->xdig_rows;
        ha.n_by = 1;
        ha.logits = a.out;
        ha.keys = a.keys;
        ha.counter = a.counter;
        ha.argmax_out = a.argmax_out;
        ha.last_tok = a.last_tok;
        ha.meta = a.meta;
        ha.err = a.err;
        ha.xsum = h->xsum;
        ha.thr = h->head_thr;
        if (int8_head) {
            // coarse logits go to the caller's buffer, or to the handle's when there is none
            if (ha.logits == nullptr) ha.logits = h->head_logits;
            e = head_int8_launch(h->num_sms, ha, h->wdig, h->xdig, h->head_cand, h->head_counter + 2,
                                 h->head_counter + 1, st);
            if (e != cudaSuccess) return cuda_fail(h, e, "int8 head launch");
            return DEC_OK;
        }
        e = head_tc_launch(h->num_sms, ha, own ? PRO : kHeadXExternal, st);
        if (e != cudaSuccess) return cuda_fail(h, e, "tensor-core head launch");
        return DEC_OK;
    }
    if (mma_eligible(h, a.N, a.K, 4, a.B)) return proj_mma<float, PRO, EPI_HEAD>(h, a, h->m_head, st);
    return gemv<float, false, PRO, EPI_HEAD, MAP_ADJ>(h, a, st);
}

// 2-D TMA descriptor of a row-major [rows, cols] matrix (f32 or int8): boxes of box_rows
// rows x 128 bytes with the 128-byte swizzle, zero fill outside the matrix.
dec_status make_wmap(dec_handle* h, CUtensorMap* m, const void* w, int rows, int cols, bool f32,
                      int box_rows = kMmaBlockRows) {
    static EncodeTiledFn encode = nullptr;
    if (encode == nullptr) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr) {
            cudaGetLastError();
            return fail(h, DEC_ECUDA, "cuTensorMapEncodeTiled is not available");
        }
        encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    const int elt = f32 ? 4 : 1;
    const cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
    const cuuint64_t strides[1] = {cuuint64_t(cols) * elt};
    const cuuint32_t box[2] = {cuuint32_t(128 / elt), cuuint32_t(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                              const_cast<void*>(w), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(h, DEC_ECUDA, "cuTensorMapEncodeTiled failed (" + std::to_string(r) + ")");
    return DEC_OK;
}

dec_status attention(dec_handle* h, AttnArgs a, int B, int max_keys, int tps, cudaStream_t st) {
    thread_local int configured_dev = -1;   // attributes are per device
    if (configured_dev != h->device) {
        DEC_CUDA(h, cudaFuncSetAttribute(k_attention, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kAttnSmemBytes)));
        DEC_CUDA(h, cudaFuncSetAttribute(k_attention, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         cudaSharedmemCarveoutMaxShared));
        configured_dev = h->device;
    }
    // fixed tiles per split (a handle constant): each row's split boundaries, hence its
    // summation order, depend only on its own length
    const AttnLaunch p = attn_launch_plan(h->num_sms, B * a.H, max_keys, tps);
    a.tps = p.tps;
    a.S = p.S;
    a.stages = p.stages;
    DEC_CUDA(h, launch(k_attention, dim3(a.S, a.H, B), dim3(kAttnThreads), attn_smem_bytes(p.stages), st, a));
    return DEC_OK;
}

// Tiles per split of the handle's self- or cross-attention launches.
int tiles_per_split(const dec_handle* h, int max_keys) {
    return attn_tiles_per_split(h->cfg.n_heads * h->max_batch, max_keys);
}

GemvArgs base_args(dec_handle* h, int B) {
    GemvArgs g{};
    g.B = B;
    g.eps = h->cfg.norm_eps;
    g.meta = h->w->meta;
    g.err = h->dev_err;
    return g;
}

// Per-phase timing: an event recorded after the phase (only while timing is on).
dec_status phase_mark(dec_handle* h, cudaStream_t st, int layer, int kind) {
    if (!h->phase_timing) return DEC_OK;
    if (h->phase_n == h->phase_ev.size()) {
        cudaEvent_t e;
        DEC_CUDA(h, cudaEventCreate(&e));
        h->phase_ev.push_back(e);
        h->phase_tag.push_back({0, 0});
    }
    DEC_CUDA(h, cudaEventRecord(h->phase_ev[h->phase_n], st));
    h->phase_tag[h->phase_n] = {layer, kind};
    ++h->phase_n;
    return DEC_OK;
}

// One decoder layer for the rows of the current chain (h->w): X holds their residual rows.
dec_status layer_step(dec_handle* h, int l, int B, float* X, int max_len_plus1, cudaStream_t st) {
    const dec_config& c = h->cfg;
    const int d = c.d_model, F = c.d_ff, H = c.n_heads;
    const LayerDev& L = h->layers[l];
    float* kc = h->kc + l * h->self_layer_stride;
    float* vc = h->vc + l * h->self_layer_stride;
    // ---- q|k|v with the cache append ----
    GemvArgs g = base_args(h, B);
    g.x = X;
    g.x_ld = d;
    g.norm_w = L.n1w;
    g.norm_b = L.n1b;
    g.K = d;
    g.N = d + 2 * kv_width(c);
    g.W = L.wqkv;
    g.scale = L.sqkv;
    g.bias = L.bqkv;
    g.out = h->w->q;
    g.out_ld = d;
    g.kc = kc;
    g.vc = vc;
    g.kv = self_kv_map(h);
    g.d = d;
    g.kvd = kv_width(c);
    if (c.family == DEC_FAMILY_WHISPER) {
        DEC_TRY((gemv_whisper<PRO_LN, EPI_QKV, MAP_ADJ>(h, g, st, L, 0)));
    } else {
        g.rope = h->rope;
        DEC_TRY((gemv_qwen<PRO_RMS, EPI_QKV, MAP_ROPE>(h, g, L.m_qkv, st)));
    }
    DEC_TRY(phase_mark(h, st, l, DEC_PHASE_QKV));
    // ---- self-attention over rows 0..len ----
    AttnArgs at{};
    at.q = h->w->q;
    at.q_bstride = d;
    at.k = kc;
    at.v = vc;
    at.slot_stride = h->self_slot_stride;
    at.ld = c.max_cache_len;
    at.H = H;
    at.kv_group = H / kv_heads(c);
    at.kv = self_kv_map(h);
    at.mode = ATTN_SELF;
    at.meta = h->w->meta;
    at.out = h->w->ctx;
    at.out_bstride = d;
    at.part = h->w->part;
    at.counters = h->w->counters;
    at.err = h->dev_err;
    at.drop_first_copy = (l == 0) ? h->inject_drop : 0;
    DEC_TRY(attention(h, at, B, max_len_plus1, h->tps_self, st));
    DEC_TRY(phase_mark(h, st, l, DEC_PHASE_SELF_ATTN));
    at.drop_first_copy = 0;
    // ---- output projection + residual ----
    g = base_args(h, B);
    g.x = h->w->ctx;
    g.x_ld = d;
    g.K = d;
    g.N = d;
    g.W = L.wo;
    g.scale = L.so;
    g.bias = L.bo;
    g.out = X;
    g.out_ld = d;
    if (c.family == DEC_FAMILY_WHISPER) {
        DEC_TRY((gemv_whisper<PRO_NONE, EPI_RESID, MAP_ADJ>(h, g, st, L, 1)));
    } else {
        DEC_TRY((gemv_qwen<PRO_NONE, EPI_RESID, MAP_ADJ>(h, g, L.m_o, st)));
    }
    DEC_TRY(phase_mark(h, st, l, DEC_PHASE_O));
    if (c.family == DEC_FAMILY_WHISPER) {
        // ---- cross-attention block ----
        g = base_args(h, B);
        g.x = X;
        g.x_ld = d;
        g.norm_w = L.n2w;
        g.norm_b = L.n2b;
        g.K = d;
        g.N = d;
        g.W = L.wxq;
        g.scale = L.sxq;
        g.bias = L.bxq;
        g.out = h->w->xq;
        g.out_ld = d;
        DEC_TRY((gemv_whisper<PRO_LN, EPI_STORE, MAP_ADJ>(h, g, st, L, 2)));
        DEC_TRY(phase_mark(h, st, l, DEC_PHASE_CROSS_Q));
        at.q = h->w->xq;
        at.k = h->xkc + l * h->cross_layer_stride;
        at.v = h->xvc + l * h->cross_layer_stride;
        at.slot_stride = h->cross_slot_stride;
        at.ld = c.enc_len;
        at.mode = ATTN_CROSS;
        at.kv_group = 1;
        at.kv.table = nullptr;
        at.n_fixed = c.enc_len;
        DEC_TRY(attention(h, at, B, c.enc_len, h->tps_cross, st));
        DEC_TRY(phase_mark(h, st, l, DEC_PHASE_CROSS_ATTN));
        g = base_args(h, B);
        g.x = h->w->ctx;
        g.x_ld = d;
        g.K = d;
        g.N = d;
        g.W = L.wxo;
        g.scale = L.sxo;
        g.bias = L.bxo;
        g.out = X;
        g.out_ld = d;
        DEC_TRY((gemv_whisper<PRO_NONE, EPI_RESID, MAP_ADJ>(h, g, st, L, 3)));
        DEC_TRY(phase_mark(h, st, l, DEC_PHASE_CROSS_O));
        // ---- GELU FFN ----
        g = base_args(h, B);
        g.x = X;
        g.x_ld = d;
        g.norm_w = L.n3w;
        g.norm_b = L.n3b;
        g.K = d;
        g.N = F;
        g.W = L.w1;
        g.scale = L.s1;
        g.bias = L.b1;
        g.out = h->w->ffn;
        g.out_ld = F;
        DEC_TRY((gemv_whisper<PRO_LN, EPI_GELU, MAP_ADJ>(h, g, st, L, 4)));
        DEC_TRY(phase_mark(h, st, l, DEC_PHASE_FFN_UP));
        g = base_args(h, B);
        g.x = h->w->ffn;
        g.x_ld = F;
        g.K = F;
        g.N = d;
        g.W = L.w2;
        g.scale = L.s2;
        g.bias = L.b2;
        g.out = X;
        g.out_ld = d;
        DEC_TRY((gemv_whisper<PRO_NONE, EPI_RESID, MAP_ADJ>(h, g, st, L, 5)));
        DEC_TRY(phase_mark(h, st, l, DEC_PHASE_FFN_DOWN));
    } else {
        // ---- SwiGLU MLP ----
        g = base_args(h, B);
        g.x = X;
        g.x_ld = d;
        g.norm_w = L.n2w;
        g.K = d;
        g.N = F;
        g.W = L.wg;
        g.W2 = L.wu;
        g.scale = L.sg;
        g.scale2 = L.su;
        g.out = h->w->ffn;
        g.out_ld = F;
        DEC_TRY((gemv_qwen<PRO_RMS, EPI_SWIGLU, MAP_DUAL>(h, g, L.m_1, st)));
        DEC_TRY(phase_mark(h, st, l, DEC_PHASE_FFN_UP));
        g = base_args(h, B);
        g.x = h->w->ffn;
        g.x_ld = F;
        g.K = F;
        g.N = d;
        g.W = L.wd;
        g.scale = L.sd;
        g.out = X;
        g.out_ld = d;
        DEC_TRY((gemv_qwen<PRO_NONE, EPI_RESID, MAP_ADJ>(h, g, L.m_2, st)));
        DEC_TRY(phase_mark(h, st, l, DEC_PHASE_FFN_DOWN));
    }
    return DEC_OK;
}

// One step for the batch described in h->dmeta (already uploaded).
// head_row0 / head_rows: the rows whose logits the head computes (all by default; a prompt
// chunk needs its last row only, or none). trace: copy each layer's residual (decode steps).
// split: run the layers as chains over equal parts of the rows (chain_bounds; the metas of the
// parts uploaded too), chain 0 on st and chain c on h->side_streams[c], with no dependency
// between chains: their kernels overlap wherever the SMs allow.
dec_status run_step(dec_handle* h, int B, int max_len_plus1, float* logits, int* argmax, cudaStream_t st,
                    int head_row0 = 0, int head_rows = -1, bool trace = true, bool split = false) {
    if (head_rows < 0) head_rows = B;
    const dec_config& c = h->cfg;
    const int d = c.d_model;
    {
        thread_local int attr_dev = -1;
        DEC_CUDA(h, prefer_max_shared_once(k_embed, attr_dev));
    }
    h->w = &h->chain[0];
    h->chain[0].meta = h->dmeta;
    h->phase_n = 0;
    DEC_TRY(phase_mark(h, st, -1, 0));
    DEC_CUDA(h, launch(k_embed, dim3(B), dim3(128), 0, st, (const float*)h->tok_emb, (const float*)h->pos_emb,
                       (const StepMeta*)h->dmeta, (const int*)h->last_tok, h->x, d, h->d_table));
    DEC_TRY(phase_mark(h, st, -1, DEC_PHASE_EMBED));
    if (!split) {
        for (int l = 0; l < c.n_layers; ++l) {
            DEC_TRY(layer_step(h, l, B, h->x, max_len_plus1, st));
            if (trace && h->trace)
                DEC_CUDA(h, cudaMemcpyAsync(h->trace + static_cast<size_t>(l) * B * d, h->x, size_t(B) * d * 4,
                                            cudaMemcpyDeviceToDevice, st));
        }
    } else {
        int r0[kMaxChains + 1];
        const int n = chain_bounds(B, r0);
        DEC_CUDA(h, cudaEventRecord(h->ev_fork, st));
        for (int ci = 1; ci < n; ++ci) DEC_CUDA(h, cudaStreamWaitEvent(h->side_streams[ci], h->ev_fork, 0));
        for (int ci = 0; ci < n; ++ci) h->chain[ci].meta = h->dmeta + 1 + ci;
        dec_status r = DEC_OK;
        for (int l = 0; l < c.n_layers && r == DEC_OK; ++l)
            for (int ci = 0; ci < n && r == DEC_OK; ++ci) {
                h->w = &h->chain[ci];
                r = layer_step(h, l, r0[ci + 1] - r0[ci], h->x + static_cast<size_t>(r0[ci]) * d, max_len_plus1,
                               ci == 0 ? st : h->side_streams[ci]);
            }
        // every chain always joins, so that a capture ends with every stream joined
        h->w = &h->chain[0];
        h->chain[0].meta = h->dmeta;
        for (int ci = 1; ci < n; ++ci) {
            DEC_CUDA(h, cudaEventRecord(h->ev_join[ci], h->side_streams[ci]));
            DEC_CUDA(h, cudaStreamWaitEvent(st, h->ev_join[ci], 0));
        }
        DEC_TRY(r);
    }
    // ---- final norm + tied head + greedy argmax ----
    if (head_rows == 0) return DEC_OK;
    GemvArgs g = base_args(h, head_rows);
    g.x = h->x + static_cast<size_t>(head_row0) * d;
    g.x_ld = d;
    g.norm_w = h->final_w;
    g.norm_b = h->final_b;
    g.K = d;
    g.N = c.vocab;
    g.W = h->tok_emb;
    g.out = logits;
    g.out_ld = c.vocab;
    g.keys = h->keys;
    g.counter = h->head_counter;
    g.argmax_out = argmax;
    g.last_tok = h->last_tok;
    if (c.family == DEC_FAMILY_WHISPER) {
        DEC_TRY(head<PRO_LN>(h, g, st));
    } else {
        DEC_TRY(head<PRO_RMS>(h, g, st));
    }
    DEC_TRY(phase_mark(h, st, -1, DEC_PHASE_HEAD));
    return DEC_OK;
}

KvMap self_kv_map(const dec_handle* h) {
    KvMap m;
    m.heads = kv_heads(h->cfg);
    if (h->page_rows > 0) {
        m.table = h->d_table;
        m.page_rows = h->page_rows;
        m.pages_per_slot = h->pages_per_slot;
    } else {
        m.table = nullptr;
        m.page_rows = h->cfg.max_cache_len;
        m.pages_per_slot = 1;
    }
    return m;
}

// Pages a slot needs beyond those it holds to keep `rows` rows (0 for a dense cache).
int pages_short(const dec_handle* h, int slot, int rows) {
    if (h->page_rows <= 0) return 0;
    const int want = (rows + h->page_rows - 1) / h->page_rows;
    return std::max(0, want - static_cast<int>(h->slot_pages[slot].size()));
}

// Give `slot` pages for `rows` rows, recording the table entries in m (applied on the device by
// the step's first kernel); the caller has checked that the pool holds enough.
void grow_slot(dec_handle* h, int slot, int rows, StepMeta& m) {
    if (h->page_rows <= 0) return;
    auto& pg = h->slot_pages[slot];
    const int want = (rows + h->page_rows - 1) / h->page_rows;
    while (static_cast<int>(pg.size()) < want) {
        const int page = h->free_pages.back();
        h->free_pages.pop_back();
        m.upd_idx[m.n_upd] = slot * h->pages_per_slot + static_cast<int>(pg.size());
        m.upd_page[m.n_upd] = page;
        ++m.n_upd;
        pg.push_back(page);
    }
}

// Return the pages of `slot` beyond those `rows` rows need to the pool.
void shrink_slot(dec_handle* h, int slot, int rows) {
    if (h->page_rows <= 0) return;
    auto& pg = h->slot_pages[slot];
    const int keep = (rows + h->page_rows - 1) / h->page_rows;
    while (static_cast<int>(pg.size()) > keep) {
        h->free_pages.push_back(pg.back());
        pg.pop_back();
    }
}

// Upload the step description through the pinned ring.
// With split, the rows of each chain follow as metas of their own (rows renumbered from 0;
// page-table updates stay with the whole step's meta, which k_embed applies).
dec_status upload_meta(dec_handle* h, const StepMeta& m, cudaStream_t st, bool split = false) {
    const int i = h->ring;
    h->ring = (h->ring + 1) % kMetaRing;
    DEC_CUDA(h, cudaEventSynchronize(h->hev[i]));
    std::memcpy(h->hmeta[i], &m, sizeof(StepMeta));
    int n_parts = 0;
    if (split) {
        int rb[kMaxChains + 1];
        n_parts = chain_bounds(m.B, rb);
        for (int ci = 0; ci < n_parts; ++ci) {
            StepMeta& o = h->hmeta[i][1 + ci];
            const int r0 = rb[ci], n = rb[ci + 1] - rb[ci];
            o.B = n;
            o.n_upd = 0;
            for (int b = 0; b < n; ++b) {
                o.slot[b] = m.slot[r0 + b];
                o.tok[b] = m.tok[r0 + b];
                o.pos[b] = m.pos[r0 + b];
                o.len[b] = m.len[r0 + b];
                o.fresh[b] = m.fresh[r0 + b];
            }
        }
    }
    DEC_CUDA(h, cudaMemcpyAsync(h->dmeta, h->hmeta[i], (1 + n_parts) * sizeof(StepMeta), cudaMemcpyHostToDevice,
                                st));
    DEC_CUDA(h, cudaEventRecord(h->hev[i], st));
    return DEC_OK;
}

// Entry points that queue work refuse it after a bounded device wait gave up, until dec_reset.
dec_status check_not_failed(dec_handle* h) {
    if (h->failed)
        return fail(h, DEC_ETIMEOUT, "a bounded device wait gave up in an earlier call; call dec_reset first");
    return DEC_OK;
}

dec_status check_device(dec_handle* h) {
    int cur = -1;
    DEC_CUDA(h, cudaGetDevice(&cur));
    if (cur != h->device) return fail(h, DEC_EINVAL, "the current CUDA device is not the handle's device");
    return DEC_OK;
}

dec_status validate_step(dec_handle* h, int B, const int32_t* slots, const int32_t* tokens,
                         const int32_t* positions, const int32_t* cache_lens, StepMeta& m, int& max_len) {
    const dec_config& c = h->cfg;
    if (B < 1 || B > h->max_batch)
        return fail(h, DEC_EINVAL, "batch must be in [1, " + std::to_string(h->max_batch) + "]");
    if (!positions || !cache_lens) return fail(h, DEC_EINVAL, "positions and cache_lens are required");
    std::vector<char> seen(c.max_slots, 0);
    m.B = B;
    max_len = 0;
    for (int b = 0; b < B; ++b) {
        const int s = slots ? slots[b] : b;
        if (s < 0 || s >= c.max_slots) return fail(h, DEC_EINVAL, "slot out of range");
        if (seen[s]) return fail(h, DEC_EINVAL, "duplicate slot in batch");
        seen[s] = 1;
        if (tokens) {
            if (tokens[b] < 0 || tokens[b] >= c.vocab)
                return fail(h, DEC_ERANGE, "token " + std::to_string(tokens[b]) + " outside [0, vocab)");
        } else if (!h->has_tok[s]) {
            return fail(h, DEC_ESTATE, "slot " + std::to_string(s) + " has no previous greedy pick");
        }
        if (positions[b] < 0 || positions[b] >= c.max_pos)
            return fail(h, DEC_ERANGE, "position " + std::to_string(positions[b]) + " outside [0, max_pos)");
        if (cache_lens[b] != h->slot_len[s])
            return fail(h, DEC_ESTATE, "cache_lens[" + std::to_string(b) + "] = " + std::to_string(cache_lens[b]) +
                                           " but slot " + std::to_string(s) + " holds " +
                                           std::to_string(h->slot_len[s]) + " rows");
        if (cache_lens[b] + 1 > c.max_cache_len)
            return fail(h, DEC_EOVERFLOW, "cache overflow: " + std::to_string(cache_lens[b]) + " + 1 > " +
                                              std::to_string(c.max_cache_len));
        if (c.family == DEC_FAMILY_WHISPER && !h->has_cross[s])
            return fail(h, DEC_ESTATE, "slot " + std::to_string(s) + " has no cross-attention K/V (prefill it)");
        m.slot[b] = s;
        m.tok[b] = tokens ? tokens[b] : -1;
        m.pos[b] = positions[b];
        m.len[b] = cache_lens[b];
        m.fresh[b] = cache_lens[b];
        max_len = std::max(max_len, cache_lens[b] + 1);
    }
    // a paged cache must have a free page for every slot whose new row starts one
    int short_pages = 0;
    for (int b = 0; b < B; ++b) short_pages += pages_short(h, m.slot[b], m.len[b] + 1);
    if (short_pages > static_cast<int>(h->free_pages.size()))
        return fail(h, DEC_ENOMEM, "KV page pool exhausted: the step needs " + std::to_string(short_pages) +
                                       " new pages, " + std::to_string(h->free_pages.size()) + " are free");
    return DEC_OK;
}

// Two-chain steps: every kernel but the attention gets the device's highest launch priority,
// so that when an SM frees up, the chain in its latency-bound projection phase gets it
// before the other chain's next attention CTA (the attention streams HBM with whatever SMs
// it holds). Best effort: a failure leaves the default priorities.
void prioritise_latency_kernels(cudaGraph_t g) {
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) {
        cudaGetLastError();
        return;
    }
    size_t n = 0;
    if (cudaGraphGetNodes(g, nullptr, &n) != cudaSuccess || n == 0) {
        cudaGetLastError();
        return;
    }
    std::vector<cudaGraphNode_t> nodes(n);
    if (cudaGraphGetNodes(g, nodes.data(), &n) != cudaSuccess) {
        cudaGetLastError();
        return;
    }
    for (auto nd : nodes) {
        cudaGraphNodeType t;
        cudaKernelNodeParams kp;
        if (cudaGraphNodeGetType(nd, &t) != cudaSuccess || t != cudaGraphNodeTypeKernel ||
            cudaGraphKernelNodeGetParams(nd, &kp) != cudaSuccess)
            continue;
        cudaKernelNodeAttrValue v{};
        v.priority = kp.func == reinterpret_cast<void*>(k_attention) ? least : greatest;
        cudaGraphKernelNodeSetAttribute(nd, cudaLaunchAttributePriority, &v);
    }
    cudaGetLastError();
}

// Record the step's launch sequence into a graph for later identical steps. Capture
// problems are not errors: the key is marked and such steps keep running eagerly.
void capture_step(dec_handle* h, const std::array<long long, 5>& key, int B, int max_len, float* logits,
                  int* argmax, bool split) {
    if (h->graphs.size() >= 256) {
        for (auto& kv : h->graphs)
            if (kv.second.exec) cudaGraphExecDestroy(kv.second.exec);
        h->graphs.clear();
    }
    cudaGraphExec_t exec = nullptr;
    int kernels = -1;
    if (cudaStreamBeginCapture(h->cap_stream, cudaStreamCaptureModeThreadLocal) == cudaSuccess) {
        const std::string saved = h->err;
        const dec_status s = run_step(h, B, max_len, logits, argmax, h->cap_stream, 0, -1, true, split);
        cudaGraph_t g = nullptr;
        const cudaError_t e = cudaStreamEndCapture(h->cap_stream, &g);
        if (s == DEC_OK && e == cudaSuccess && g != nullptr) {
            if (split) prioritise_latency_kernels(g);
            if (cudaGraphInstantiate(&exec, g, 0) != cudaSuccess) exec = nullptr;
            size_t n = 0;
            if (exec && cudaGraphGetNodes(g, nullptr, &n) == cudaSuccess) {
                std::vector<cudaGraphNode_t> nodes(n);
                if (n && cudaGraphGetNodes(g, nodes.data(), &n) == cudaSuccess) {
                    kernels = 0;
                    for (auto nd : nodes) {
                        cudaGraphNodeType t;
                        if (cudaGraphNodeGetType(nd, &t) == cudaSuccess && t == cudaGraphNodeTypeKernel) ++kernels;
                    }
                }
            }
        }
        if (g) cudaGraphDestroy(g);
        h->err = saved;
    }
    cudaGetLastError();
    h->graphs[key] = {exec, kernels};
}

dec_status step_validated(dec_handle* h, StepMeta& m, int max_len, float* logits, int* argmax,
                          cudaStream_t st) {
    m.n_upd = 0;
    for (int b = 0; b < m.B; ++b) grow_slot(h, m.slot[b], m.len[b] + 1, m);
    // two chains for large batches, unless per-layer copies, phase timing or fault injection
    // need the single launch sequence
    const bool split =
        h->n_chains > 1 && m.B >= kSplitMinBatch && !h->trace && !h->phase_timing && !h->inject_drop;
    DEC_TRY(upload_meta(h, m, st, split));
    const std::array<long long, 5> key = {m.B, (max_len + kAttnTile - 1) / kAttnTile,
                                          reinterpret_cast<long long>(logits), reinterpret_cast<long long>(argmax),
                                          reinterpret_cast<long long>(h->trace)};
    auto it = h->graphs.find(key);
    if (h->inject_drop || h->phase_timing) {
        // fault-injection and phase-timed steps run eagerly and are never captured
        DEC_TRY(run_step(h, m.B, max_len, logits, argmax, st));
        h->last_step_kernels = -1;
    } else if (it != h->graphs.end() && it->second.exec != nullptr) {
        DEC_CUDA(h, cudaGraphLaunch(it->second.exec, st));
        h->last_step_kernels = it->second.kernels;
    } else {
        DEC_TRY(run_step(h, m.B, max_len, logits, argmax, st, 0, -1, true, split));
        if (it == h->graphs.end()) capture_step(h, key, m.B, max_len, logits, argmax, split);
        h->last_step_kernels = h->graphs[key].kernels;
    }
    for (int b = 0; b < m.B; ++b) {
        h->slot_len[m.slot[b]] += 1;
        h->has_tok[m.slot[b]] = 1;
    }
    h->last_batch = m.B;
    return DEC_OK;
}

}  // namespace

// ===================================================================== C ABI

extern "C" {

const char* dec_last_error(const dec_handle* h) { return h ? h->err.c_str() : g_create_error.c_str(); }

dec_status dec_destroy(dec_handle* h) {
    if (!h) return DEC_OK;
    cudaDeviceSynchronize();
    for (auto& kv : h->graphs)
        if (kv.second.exec) cudaGraphExecDestroy(kv.second.exec);
    for (cudaEvent_t e : h->phase_ev) cudaEventDestroy(e);
    if (h->cap_stream) cudaStreamDestroy(h->cap_stream);
    for (int ci = 1; ci < kMaxChains; ++ci) {
        if (h->side_streams[ci]) cudaStreamDestroy(h->side_streams[ci]);
        if (h->ev_join[ci]) cudaEventDestroy(h->ev_join[ci]);
    }
    if (h->ev_fork) cudaEventDestroy(h->ev_fork);
    for (void* p : h->dallocs) cudaFree(p);
    for (void* p : h->hallocs) cudaFreeHost(p);
    for (int i = 0; i < kMetaRing; ++i)
        if (h->hev[i]) cudaEventDestroy(h->hev[i]);
    delete h;
    return DEC_OK;
}

static dec_status create_impl(dec_handle* h, const dec_config* cfg, const dec_weights* w) {
    const dec_config& c = *cfg;
    const int d = c.d_model, F = c.d_ff, H = c.n_heads, L = c.n_layers;
    const bool wh = c.family == DEC_FAMILY_WHISPER;
    DEC_CUDA(h, cudaGetDevice(&h->device));
    DEC_CUDA(h, cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device));
    if (!w->tok_emb || !w->final_w || !w->layers) return fail(h, DEC_EINVAL, "missing embedding, final norm or layers");
    if (wh && (!w->pos_emb || !w->final_b)) return fail(h, DEC_EINVAL, "whisper needs pos_emb and final_b");
    DEC_TRY(upload(h, &h->tok_emb, w->tok_emb, size_t(c.vocab) * d * 4));
    if (wh) {
        DEC_TRY(upload(h, &h->pos_emb, w->pos_emb, size_t(c.max_pos) * d * 4));
        DEC_TRY(upload(h, &h->final_b, w->final_b, size_t(d) * 4));
    } else {
        DEC_TRY(build_rope(h));
    }
    DEC_TRY(upload(h, &h->final_w, w->final_w, size_t(d) * 4));
    h->layers.resize(L);
    for (int l = 0; l < L; ++l) {
        const dec_layer_weights& W = w->layers[l];
        LayerDev& D = h->layers[l];
        if (!W.norm1_w || !W.norm2_w) return fail(h, DEC_EINVAL, "missing norm weights");
        DEC_TRY(upload(h, &D.n1w, W.norm1_w, size_t(d) * 4));
        DEC_TRY(upload(h, &D.n2w, W.norm2_w, size_t(d) * 4));
        DEC_TRY(upload_qkv(h, W, D));
        if (wh) {
            if (!W.norm1_b || !W.norm2_b || !W.norm3_w || !W.norm3_b)
                return fail(h, DEC_EINVAL, "missing layer norm parameters");
            DEC_TRY(upload(h, &D.n1b, W.norm1_b, size_t(d) * 4));
            DEC_TRY(upload(h, &D.n2b, W.norm2_b, size_t(d) * 4));
            DEC_TRY(upload(h, &D.n3w, W.norm3_w, size_t(d) * 4));
            DEC_TRY(upload(h, &D.n3b, W.norm3_b, size_t(d) * 4));
            DEC_TRY(upload_proj(h, W.o, d, d, true, &D.wo, &D.so, &D.bo, "o"));
            DEC_TRY(upload_proj(h, W.xq, d, d, true, &D.wxq, &D.sxq, &D.bxq, "xq"));
            DEC_TRY(upload_proj(h, W.xk, d, d, true, &D.wxk, &D.sxk, &D.bxk, "xk"));
            DEC_TRY(upload_proj(h, W.xv, d, d, true, &D.wxv, &D.sxv, &D.bxv, "xv"));
            DEC_TRY(upload_proj(h, W.xo, d, d, true, &D.wxo, &D.sxo, &D.bxo, "xo"));
            DEC_TRY(upload_proj(h, W.fc1, F, d, true, &D.w1, &D.s1, &D.b1, "fc1"));
            DEC_TRY(upload_proj(h, W.fc2, d, F, true, &D.w2, &D.s2, &D.b2, "fc2"));
        } else {
            DEC_TRY(upload_proj(h, W.o, d, d, false, &D.wo, &D.so, &D.bo, "o"));
            float* nobias = nullptr;
            DEC_TRY(upload_proj(h, W.gate, F, d, false, &D.wg, &D.sg, &nobias, "gate"));
            DEC_TRY(upload_proj(h, W.up, F, d, false, &D.wu, &D.su, &nobias, "up"));
            DEC_TRY(upload_proj(h, W.down, d, F, false, &D.wd, &D.sd, &nobias, "down"));
        }
    }
    // TMA descriptors of the tensor-core projection path (the head, every projection);
    // without them the CUDA-core kernels run instead. The Qwen q|k|v and gate/up panels
    // get row-permuted copies for the int8 kernel's RoPE and SwiGLU row maps.
    {
        const bool f32w = c.proj_fmt == DEC_PROJ_F32;
        dec_status ts = make_wmap(h, &h->m_head, h->tok_emb, c.vocab, d, true);
        for (int l = 0; l < L && ts == DEC_OK; ++l) {
            LayerDev& D = h->layers[l];
            if (wh) {
                ts = make_wmap(h, &D.m_qkv, D.wqkv, d + 2 * kv_width(c), d, f32w);
                if (ts == DEC_OK) ts = make_wmap(h, &D.m_o, D.wo, d, d, f32w);
                if (ts == DEC_OK) ts = make_wmap(h, &D.m_xq, D.wxq, d, d, f32w);
                if (ts == DEC_OK) ts = make_wmap(h, &D.m_xo, D.wxo, d, d, f32w);
                if (ts == DEC_OK) ts = make_wmap(h, &D.m_1, D.w1, F, d, f32w);
                if (ts == DEC_OK) ts = make_wmap(h, &D.m_2, D.w2, d, F, f32w);
            } else {
                const int qkv_rows = d + 2 * kv_width(c);
                DEC_TRY(dalloc(h, &D.wqkv_p, size_t(qkv_rows) * d));
                DEC_TRY(dalloc(h, &D.wgu, size_t(2) * F * d));
                DEC_CUDA(h, tc_rows_permute(MAP_ROPE, static_cast<int8_t*>(D.wqkv_p),
                                            static_cast<const int8_t*>(D.wqkv), nullptr, qkv_rows, d, 0));
                DEC_CUDA(h, tc_rows_permute(MAP_DUAL, static_cast<int8_t*>(D.wgu), static_cast<const int8_t*>(D.wg),
                                            static_cast<const int8_t*>(D.wu), 2 * F, d, 0));
                ts = make_wmap(h, &D.m_qkv, D.wqkv_p, qkv_rows, d, false);
                if (ts == DEC_OK) ts = make_wmap(h, &D.m_o, D.wo, d, d, false);
                if (ts == DEC_OK) ts = make_wmap(h, &D.m_1, D.wgu, 2 * F, d, false);
                if (ts == DEC_OK) ts = make_wmap(h, &D.m_2, D.wd, d, F, false);
            }
        }
        h->tma_ok = (ts == DEC_OK);
        if (!h->tma_ok) h->err.clear();
    }
    // tcgen05 head: the embedding's digit planes (once) and the hidden rows' buffers
    if (h->tma_ok && head_tc_stages(d, 32) > 0) {
        const long long V = c.vocab;
        DEC_TRY(dalloc(h, &h->wdig, size_t(3) * V * d));
        DEC_TRY(dalloc(h, &h->wsc, size_t(V) * 4));
        DEC_CUDA(h, rowprep_digits_launch<PRO_NONE>(h->tok_emb, d, nullptr, nullptr, 0.0f, d, c.vocab, V * d, h->wdig,
                                                   h->wsc, nullptr, false, 0));
        h->xdig_rows = std::max(std::min(c.max_slots, DEC_MAX_BATCH), 32);
        const size_t xb = size_t(3) * h->xdig_rows * d;
        DEC_TRY(dalloc(h, &h->xdig, xb));
        DEC_CUDA(h, cudaMemset(h->xdig, 0, xb));
        DEC_TRY(dalloc(h, &h->xsc, size_t(h->xdig_rows) * 4));
        DEC_CUDA(h, cudaMemset(h->xsc, 0, size_t(h->xdig_rows) * 4));
        DEC_TRY(dalloc(h, &h->xsum, size_t(h->xdig_rows) * 8));
        DEC_CUDA(h, cudaMemset(h->xsum, 0, size_t(h->xdig_rows) * 8));
        if (c.head_fmt == DEC_HEAD_INT8_REFINE) {
            const size_t mb = size_t(std::min(c.max_slots, DEC_MAX_BATCH));
            DEC_TRY(dalloc(h, &h->head_thr, mb * 4));
            DEC_TRY(dalloc(h, &h->head_cand, mb * size_t(c.vocab) * 4));
            DEC_TRY(dalloc(h, &h->head_logits, mb * size_t(c.vocab) * 4));
        }
        dec_status ts = make_wmap(h, &h->m_wdig, h->wdig, int(3 * V), d, false);
        if (ts == DEC_OK) ts = make_wmap(h, &h->m_xdig16, h->xdig, 3 * h->xdig_rows, d, false, 16);
        if (ts == DEC_OK) ts = make_wmap(h, &h->m_xdig32, h->xdig, 3 * h->xdig_rows, d, false, 32);
        h->head_tc_ok = (ts == DEC_OK);
        if (!h->head_tc_ok) h->err.clear();
        if (!h->head_tc_ok && c.head_fmt == DEC_HEAD_INT8_REFINE)
            return fail(h, DEC_EINVAL, "the int8 head needs the tensor-core head (TMA descriptors unavailable)");
        DEC_CUDA(h, cudaDeviceSynchronize());
    }
    // caches
    h->self_slot_stride = (long long)kv_heads(c) * c.max_cache_len * 64;
    h->self_layer_stride = h->self_slot_stride * c.max_slots;
    h->slot_pages.assign(c.max_slots, {});
    if (c.kv_page_rows > 0) {
        h->page_rows = c.kv_page_rows;
        h->pages_per_slot = (c.max_cache_len + c.kv_page_rows - 1) / c.kv_page_rows;
        h->n_pages = c.kv_pages;
        h->self_layer_stride = (long long)c.kv_pages * kv_heads(c) * c.kv_page_rows * 64;
        DEC_TRY(dalloc(h, &h->d_table, size_t(c.max_slots) * h->pages_per_slot * 4));
        DEC_CUDA(h, cudaMemset(h->d_table, 0, size_t(c.max_slots) * h->pages_per_slot * 4));
        for (int pg = c.kv_pages - 1; pg >= 0; --pg) h->free_pages.push_back(pg);   // page 0 first
    }
    const size_t self_bytes = size_t(L) * h->self_layer_stride * 4;
    DEC_TRY(dalloc(h, &h->kc, self_bytes));
    DEC_TRY(dalloc(h, &h->vc, self_bytes));
    DEC_CUDA(h, cudaMemset(h->kc, 0, self_bytes));
    DEC_CUDA(h, cudaMemset(h->vc, 0, self_bytes));
    if (wh) {
        h->cross_slot_stride = (long long)H * c.enc_len * 64;
        h->cross_layer_stride = h->cross_slot_stride * c.max_slots;
        const size_t cross_bytes = size_t(L) * h->cross_layer_stride * 4;
        DEC_TRY(dalloc(h, &h->xkc, cross_bytes));
        DEC_TRY(dalloc(h, &h->xvc, cross_bytes));
    }
    // workspace
    h->max_batch = std::min(c.max_slots, DEC_MAX_BATCH);
    h->tps_self = tiles_per_split(h, c.max_cache_len);
    h->tps_cross = wh ? tiles_per_split(h, c.enc_len) : 1;
    // per-step workspaces hold a decode batch or a prompt chunk, whichever is larger
    h->max_rows = std::max(h->max_batch, kPrefillChunk);
    const int MB = h->max_rows;
    DEC_TRY(dalloc(h, &h->x, size_t(MB) * d * 4));
    // Whisper W8A32, tcgen05 path: the activation digit planes (per chain, below)
    bool digit_maps_ok = h->tma_ok && wh && c.proj_fmt == DEC_PROJ_W8A32;
    // split-K scratch of the largest tensor-core plan
    size_t pb = 16;
    int cl = 1;
    if (h->tma_ok) {
        const int welt = c.proj_fmt == DEC_PROJ_F32 ? 4 : 1;
        auto need_f32 = [&](int n, int k, int elt) {
            const MmaPlan p = mma_plan(n, k, elt, h->num_sms);
            if (!p.ok) return;
            pb = std::max(pb, mma_part_bytes(p, MB));
            cl = std::max(cl, mma_counters(p, MB));
        };
        auto need_i8 = [&](int n, int k) {
            const MmaPlan p = tc_plan(n, k, h->num_sms);
            if (!p.ok) return;
            pb = std::max(pb, tc_part_bytes(p, MB));
            cl = std::max(cl, tc_counters(p, MB));
        };
        auto need_digits = [&](int n, int k) {
            const MmaPlan p = tc_plan(n, k, h->num_sms, 3);
            if (!p.ok) return;
            pb = std::max(pb, tc_part_bytes(p, MB, 3));
            cl = std::max(cl, tc_counters(p, MB));
        };
        need_f32(c.vocab, d, 4);
        const int shapes[4][2] = {{d + 2 * kv_width(c), d}, {d, d}, {F, d}, {d, F}};
        for (const auto& sh : shapes) {
            if (!wh) {
                need_i8(sh[0] == F ? 2 * F : sh[0], sh[1]);
            } else {
                need_f32(sh[0], sh[1], welt);
                if (welt == 1) need_digits(sh[0], sh[1]);
            }
        }
    }
    // per-chain scratch: chain 0 always, chain 1 when decode batches can be split in two
    {
        int rb[kMaxChains + 1];
        h->n_chains = h->max_batch >= kSplitMinBatch ? chain_bounds(h->max_batch, rb) : 1;
    }
    for (int ci = 0; ci < h->n_chains; ++ci) {
        Chain& ch = h->chain[ci];
        DEC_TRY(dalloc(h, &ch.q, size_t(MB) * d * 4));
        DEC_TRY(dalloc(h, &ch.ctx, size_t(MB) * d * 4));
        DEC_TRY(dalloc(h, &ch.xq, size_t(MB) * d * 4));
        DEC_TRY(dalloc(h, &ch.ffn, size_t(MB) * F * 4));
        DEC_TRY(dalloc(h, &ch.part, size_t(MB) * H * kMaxSplits * kAttnPartStride * 4));
        DEC_TRY(dalloc(h, &ch.counters, size_t(MB) * H * 4));
        DEC_CUDA(h, cudaMemset(ch.counters, 0, size_t(MB) * H * 4));
        if (!h->tma_ok) continue;
        // tensor-core path: normalised / quantised rows and the split-K scratch
        DEC_TRY(dalloc(h, &ch.xn, size_t(MB) * std::max(d, F) * 4));
        ch.xq8_rows = std::max(MB, 32);
        DEC_TRY(dalloc(h, &ch.xq8, size_t(ch.xq8_rows) * std::max(d, F)));
        DEC_CUDA(h, cudaMemset(ch.xq8, 0, size_t(ch.xq8_rows) * std::max(d, F)));
        const int ks[2] = {d, F};
        if (!wh)
            for (int i = 0; i < 2; ++i)
                for (int j = 0; j < 2; ++j)
                    DEC_TRY(make_wmap(h, &ch.m_xq8[i][j], ch.xq8, ch.xq8_rows, ks[i], false, j ? 32 : 16));
        DEC_TRY(dalloc(h, &ch.xs8, size_t(MB) * 4));
        if (digit_maps_ok) {
            // Whisper tcgen05 path: the activation rows' digit planes
            ch.xd_rows = ((std::max(MB, 32) + 31) / 32) * 32;
            const size_t xb = size_t(3) * ch.xd_rows * std::max(d, F);
            DEC_TRY(dalloc(h, &ch.xd3, xb));
            DEC_CUDA(h, cudaMemset(ch.xd3, 0, xb));
            DEC_TRY(dalloc(h, &ch.xsd, size_t(ch.xd_rows) * 4));
            DEC_CUDA(h, cudaMemset(ch.xsd, 0, size_t(ch.xd_rows) * 4));
            dec_status ts = DEC_OK;
            for (int i = 0; i < 2 && ts == DEC_OK; ++i)
                for (int j = 0; j < 2 && ts == DEC_OK; ++j)
                    ts = make_wmap(h, &ch.m_xd3[i][j], ch.xd3, 3 * ch.xd_rows, ks[i], false, j ? 32 : 16);
            if (ts != DEC_OK) {
                digit_maps_ok = false;
                h->err.clear();
            }
        }
        DEC_TRY(dalloc(h, &ch.mma_part, pb));
        ch.mma_part_bytes = pb;
        DEC_TRY(dalloc(h, &ch.mma_cnt, size_t(cl) * 4));
        DEC_CUDA(h, cudaMemset(ch.mma_cnt, 0, size_t(cl) * 4));
        ch.mma_cnt_len = cl;
    }
    h->tcd_ok = digit_maps_ok;
    DEC_TRY(dalloc(h, &h->keys, size_t(MB) * 8));
    DEC_CUDA(h, cudaMemset(h->keys, 0, size_t(MB) * 8));
    DEC_TRY(dalloc(h, &h->head_counter, 16));
    DEC_CUDA(h, cudaMemset(h->head_counter, 0, 16));
    DEC_TRY(dalloc(h, &h->last_tok, size_t(c.max_slots) * 4));
    DEC_CUDA(h, cudaMemset(h->last_tok, 0, size_t(c.max_slots) * 4));
    DEC_TRY(dalloc(h, &h->dev_err, kStatusWords * 4));
    DEC_CUDA(h, cudaMemset(h->dev_err, 0, kStatusWords * 4));
    DEC_TRY(dalloc(h, &h->dmeta, (1 + kMaxChains) * sizeof(StepMeta)));
    h->chain[0].meta = h->dmeta;
    if (h->n_chains > 1) {
        DEC_CUDA(h, cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming));
        for (int ci = 1; ci < h->n_chains; ++ci) {
            DEC_CUDA(h, cudaStreamCreateWithFlags(&h->side_streams[ci], cudaStreamNonBlocking));
            DEC_CUDA(h, cudaEventCreateWithFlags(&h->ev_join[ci], cudaEventDisableTiming));
        }
    }
    DEC_TRY(dalloc(h, &h->stage_logits, size_t(h->max_batch) * c.vocab * 4));
    DEC_TRY(dalloc(h, &h->stage_argmax, size_t(h->max_batch) * 4));
    auto halloc = [&](void** p, size_t bytes) {
        if (injected_alloc_failure()) return fail(h, DEC_ENOMEM, "cudaMallocHost failed (injected)");
        if (cudaMallocHost(p, bytes) != cudaSuccess) {
            cudaGetLastError();
            return fail(h, DEC_ENOMEM, "cudaMallocHost failed");
        }
        h->hallocs.push_back(*p);
        return DEC_OK;
    };
    for (int i = 0; i < kMetaRing; ++i) {
        void* p = nullptr;
        DEC_TRY(halloc(&p, (1 + kMaxChains) * sizeof(StepMeta)));
        h->hmeta[i] = static_cast<StepMeta*>(p);
        DEC_CUDA(h, cudaEventCreateWithFlags(&h->hev[i], cudaEventDisableTiming));
    }
    {
        void* p = nullptr;
        DEC_TRY(halloc(&p, 16));
        h->host_status = static_cast<int*>(p);
        *h->host_status = 0;
        DEC_TRY(halloc(&p, size_t(c.max_slots) * 4));
        h->host_tok = static_cast<int*>(p);
    }
    DEC_CUDA(h, cudaStreamCreateWithFlags(&h->cap_stream, cudaStreamNonBlocking));
    h->slot_len.assign(c.max_slots, 0);
    h->has_tok.assign(c.max_slots, 0);
    h->has_cross.assign(c.max_slots, 0);
    DEC_CUDA(h, cudaDeviceSynchronize());
    return DEC_OK;
}

dec_status dec_create(const dec_config* cfg, const dec_weights* w, dec_handle** out) {
    g_create_error.clear();
    if (!out) return fail(nullptr, DEC_EINVAL, "out is NULL");
    *out = nullptr;
    if (!cfg || !w) return fail(nullptr, DEC_EINVAL, "cfg and weights are required");
    dec_status st = validate_config(*cfg);
    if (st != DEC_OK) return st;
    dec_handle* h = new dec_handle();
    h->cfg = *cfg;
    g_alloc_count = 0;
    st = create_impl(h, cfg, w);
    g_fail_alloc_at = 0;   // the hook covers one dec_create
    if (st != DEC_OK) {
        g_create_error = h->err;
        dec_destroy(h);
        return st;
    }
    *out = h;
    return DEC_OK;
}

dec_status dec_prefill(dec_handle* h, int32_t slot, const int32_t* tokens, int32_t n_tokens,
                       const float* enc_hidden, float* last_logits, void* stream) {
    if (!h) return DEC_EINVAL;
    DEC_TRY(check_not_failed(h));
    const dec_config& c = h->cfg;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (slot < 0 || slot >= c.max_slots) return fail(h, DEC_EINVAL, "slot out of range");
    if (n_tokens < 0 || (n_tokens > 0 && !tokens)) return fail(h, DEC_EINVAL, "bad tokens");
    if (n_tokens > c.max_cache_len) return fail(h, DEC_EOVERFLOW, "prefill longer than max_cache_len");
    if (c.family == DEC_FAMILY_WHISPER) {
        if (!enc_hidden) return fail(h, DEC_EINVAL, "whisper prefill needs enc_hidden");
        if (n_tokens > c.max_pos) return fail(h, DEC_ERANGE, "prefill longer than the position table");
    } else if (enc_hidden) {
        return fail(h, DEC_EINVAL, "qwen2 has no cross-attention; enc_hidden must be NULL");
    }
    for (int i = 0; i < n_tokens; ++i)
        if (tokens[i] < 0 || tokens[i] >= c.vocab) return fail(h, DEC_ERANGE, "token outside [0, vocab)");
    if (h->page_rows > 0) {
        const int need = (n_tokens + h->page_rows - 1) / h->page_rows;
        const int avail = static_cast<int>(h->free_pages.size() + h->slot_pages[slot].size());
        if (need > avail)
            return fail(h, DEC_ENOMEM, "KV page pool exhausted: the prompt needs " + std::to_string(need) +
                                           " pages, " + std::to_string(avail) + " are available");
    }
    DEC_TRY(check_device(h));
    if (c.family == DEC_FAMILY_WHISPER) {
        const int d = c.d_model;
        for (int l = 0; l < c.n_layers; ++l) {
            const LayerDev& L = h->layers[l];
            float* ko = h->xkc + l * h->cross_layer_stride + slot * h->cross_slot_stride;
            float* vo = h->xvc + l * h->cross_layer_stride + slot * h->cross_slot_stride;
            dim3 grid((d + 63) / 64, (c.enc_len + 63) / 64);
            if (c.proj_fmt == DEC_PROJ_F32) {
                k_cross_kv<float><<<grid, 256, 0, st>>>(enc_hidden, (const float*)L.wxk, nullptr, L.bxk, ko, c.enc_len, d, d);
                k_cross_kv<float><<<grid, 256, 0, st>>>(enc_hidden, (const float*)L.wxv, nullptr, L.bxv, vo, c.enc_len, d, d);
            } else {
                k_cross_kv<int8_t><<<grid, 256, 0, st>>>(enc_hidden, (const int8_t*)L.wxk, L.sxk, L.bxk, ko, c.enc_len, d, d);
                k_cross_kv<int8_t><<<grid, 256, 0, st>>>(enc_hidden, (const int8_t*)L.wxv, L.sxv, L.bxv, vo, c.enc_len, d, d);
            }
            DEC_CUDA(h, cudaGetLastError());
        }
        h->has_cross[slot] = 1;
    }
    h->slot_len[slot] = 0;
    h->has_tok[slot] = 0;
    shrink_slot(h, slot, 0);
    // The prompt runs in chunks of up to prefill_chunk rows of this one slot at consecutive
    // positions ([focr] `forward_prefill_seed`: the whole prompt in one forward): each
    // chunk is one step whose projections are m = chunk contractions and whose attention is
    // causal per row (row i attends cache rows 0..i, the chunk's earlier rows included).
    // Only the prompt's last row goes through the head. Chunks run uncaptured.
    for (int i0 = 0; i0 < n_tokens; i0 += h->prefill_chunk) {
        const int B = std::min(h->prefill_chunk, n_tokens - i0);
        StepMeta m{};
        m.B = B;
        for (int b = 0; b < B; ++b) {
            m.slot[b] = slot;
            m.tok[b] = tokens[i0 + b];
            m.pos[b] = i0 + b;
            m.len[b] = i0 + b;
            m.fresh[b] = i0;
        }
        grow_slot(h, slot, i0 + B, m);
        const bool last = i0 + B == n_tokens;
        DEC_TRY(upload_meta(h, m, st));
        const bool timing = h->phase_timing;   // prompt chunks are not phase-timed
        h->phase_timing = false;
        struct Restore {
            dec_handle* h;
            bool v;
            ~Restore() { h->phase_timing = v; }
        } restore{h, timing};
        DEC_TRY(run_step(h, B, i0 + B, last ? last_logits : nullptr, nullptr, st, B - 1, last ? 1 : 0, false));
        h->slot_len[slot] = i0 + B;
    }
    if (n_tokens > 0) h->has_tok[slot] = 1;
    h->last_batch = 0;
    return DEC_OK;
}

dec_status dec_kv_append(dec_handle* h, int32_t slot, int32_t start_pos, int32_t n_rows, const float* k,
                         const float* v, void* stream) {
    if (!h) return DEC_EINVAL;
    DEC_TRY(check_not_failed(h));
    const dec_config& c = h->cfg;
    if (slot < 0 || slot >= c.max_slots) return fail(h, DEC_EINVAL, "slot out of range");
    if (n_rows < 0 || (n_rows > 0 && (!k || !v))) return fail(h, DEC_EINVAL, "bad rows");
    if (start_pos < 0 || start_pos > h->slot_len[slot])
        return fail(h, DEC_ESTATE, "start_pos must be within [0, slot length]");
    if (start_pos + n_rows > c.max_cache_len) return fail(h, DEC_EOVERFLOW, "cache overflow");
    if (pages_short(h, slot, start_pos + n_rows) > static_cast<int>(h->free_pages.size()))
        return fail(h, DEC_ENOMEM, "KV page pool exhausted");
    DEC_TRY(check_device(h));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // pages: keep those the rows need, then add the missing ones (table entries applied on the
    // device before the copy, a step description's worth at a time)
    shrink_slot(h, slot, start_pos + n_rows);
    while (pages_short(h, slot, start_pos + n_rows) > 0) {
        StepMeta m{};
        const int have = static_cast<int>(h->slot_pages[slot].size());
        const int upto = std::min(start_pos + n_rows, (have + kMaxTableUpdates) * h->page_rows);
        grow_slot(h, slot, upto, m);
        DEC_TRY(upload_meta(h, m, st));
        k_table_update<<<1, 256, 0, st>>>(h->dmeta, h->d_table);
        DEC_CUDA(h, cudaGetLastError());
    }
    if (n_rows > 0) {
        dim3 grid(n_rows, c.n_layers);
        const KvMap km = self_kv_map(h);
        k_kv_copy<<<grid, 128, 0, st>>>(h->kc, const_cast<float*>(k), 0, h->self_layer_stride, km, slot, start_pos,
                                        n_rows, kv_width(c), 0);
        k_kv_copy<<<grid, 128, 0, st>>>(h->vc, const_cast<float*>(v), 0, h->self_layer_stride, km, slot, start_pos,
                                        n_rows, kv_width(c), 0);
        DEC_CUDA(h, cudaGetLastError());
    }
    h->slot_len[slot] = start_pos + n_rows;
    return DEC_OK;
}

dec_status dec_kv_read(dec_handle* h, int32_t slot, int32_t layer, int32_t start, int32_t n, float* k_out,
                       float* v_out, void* stream) {
    if (!h) return DEC_EINVAL;
    const dec_config& c = h->cfg;
    if (slot < 0 || slot >= c.max_slots || layer < 0 || layer >= c.n_layers)
        return fail(h, DEC_EINVAL, "slot or layer out of range");
    if (start < 0 || n < 0 || start + n > c.max_cache_len) return fail(h, DEC_EINVAL, "rows out of range");
    if (h->page_rows > 0 && start + n > static_cast<int>(h->slot_pages[slot].size()) * h->page_rows)
        return fail(h, DEC_EINVAL, "rows beyond the slot's pages");
    if (n > 0 && (!k_out || !v_out)) return fail(h, DEC_EINVAL, "null output");
    DEC_TRY(check_device(h));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (n > 0) {
        dim3 grid(n, 1);
        const KvMap km = self_kv_map(h);
        k_kv_copy<<<grid, 128, 0, st>>>(h->kc, k_out, 1, h->self_layer_stride, km, slot, start, n, kv_width(c),
                                        layer);
        k_kv_copy<<<grid, 128, 0, st>>>(h->vc, v_out, 1, h->self_layer_stride, km, slot, start, n, kv_width(c),
                                        layer);
        DEC_CUDA(h, cudaGetLastError());
    }
    return DEC_OK;
}

dec_status dec_step(dec_handle* h, int32_t batch, const int32_t* slots, const int32_t* tokens,
                    const int32_t* positions, const int32_t* cache_lens, float* logits, int32_t* argmax,
                    void* stream) {
    if (!h) return DEC_EINVAL;
    DEC_TRY(check_not_failed(h));
    StepMeta m{};
    int max_len = 0;
    DEC_TRY(validate_step(h, batch, slots, tokens, positions, cache_lens, m, max_len));
    DEC_TRY(check_device(h));
    return step_validated(h, m, max_len, logits, argmax, static_cast<cudaStream_t>(stream));
}

dec_status dec_step_host(dec_handle* h, int32_t batch, const int32_t* slots, const int32_t* tokens,
                         const int32_t* positions, const int32_t* cache_lens, float* logits_host,
                         int32_t* argmax_host, void* stream) {
    if (!h) return DEC_EINVAL;
    DEC_TRY(check_not_failed(h));
    StepMeta m{};
    int max_len = 0;
    DEC_TRY(validate_step(h, batch, slots, tokens, positions, cache_lens, m, max_len));
    DEC_TRY(check_device(h));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const dec_config& c = h->cfg;
    DEC_TRY(step_validated(h, m, max_len, logits_host ? h->stage_logits : nullptr, h->stage_argmax, st));
    if (logits_host)
        DEC_CUDA(h, cudaMemcpyAsync(logits_host, h->stage_logits, size_t(batch) * c.vocab * 4,
                                    cudaMemcpyDeviceToHost, st));
    if (argmax_host)
        DEC_CUDA(h, cudaMemcpyAsync(argmax_host, h->stage_argmax, size_t(batch) * 4, cudaMemcpyDeviceToHost, st));
    DEC_CUDA(h, cudaMemcpyAsync(h->host_status, h->dev_err, 4, cudaMemcpyDeviceToHost, st));
    DEC_CUDA(h, cudaStreamSynchronize(st));
    if (*h->host_status) {
        h->failed = true;
        return fail(h, DEC_ETIMEOUT, "a bounded device wait gave up during this step; its results are not valid");
    }
    return DEC_OK;
}

dec_status dec_slot_len(const dec_handle* h, int32_t slot, int32_t* len) {
    if (!h || !len || slot < 0 || slot >= h->cfg.max_slots) return DEC_EINVAL;
    *len = h->slot_len[slot];
    return DEC_OK;
}

dec_status dec_next_tokens(dec_handle* h, int32_t n, const int32_t* slots, int32_t* tokens, void* stream) {
    if (!h) return fail(nullptr, DEC_EINVAL, "dec_next_tokens: null handle");
    if (n < 0 || (n > 0 && (!slots || !tokens))) return fail(h, DEC_EINVAL, "dec_next_tokens: bad arguments");
    for (int i = 0; i < n; ++i) {
        if (slots[i] < 0 || slots[i] >= h->cfg.max_slots) return fail(h, DEC_EINVAL, "dec_next_tokens: slot out of range");
        if (!h->has_tok[slots[i]])
            return fail(h, DEC_ESTATE, "slot " + std::to_string(slots[i]) + " has no greedy continuation yet");
    }
    DEC_TRY(check_device(h));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    DEC_CUDA(h, cudaMemcpyAsync(h->host_tok, h->last_tok, size_t(h->cfg.max_slots) * 4, cudaMemcpyDeviceToHost, st));
    DEC_CUDA(h, cudaMemcpyAsync(h->host_status, h->dev_err, 4, cudaMemcpyDeviceToHost, st));
    DEC_CUDA(h, cudaStreamSynchronize(st));
    if (*h->host_status) {
        h->failed = true;
        return fail(h, DEC_ETIMEOUT, "a bounded device wait gave up; the tokens are not valid");
    }
    for (int i = 0; i < n; ++i) tokens[i] = h->host_tok[slots[i]];
    return DEC_OK;
}

dec_status dec_get_config(const dec_handle* h, dec_config* out) {
    if (!h || !out) return fail(nullptr, DEC_EINVAL, "dec_get_config: null pointer");
    *out = h->cfg;
    return DEC_OK;
}

dec_status dec_hidden(dec_handle* h, float* out, int32_t batch, void* stream) {
    if (!h) return DEC_EINVAL;
    if (!out || batch < 1 || batch > h->last_batch) return fail(h, DEC_EINVAL, "bad output or batch");
    DEC_CUDA(h, cudaMemcpyAsync(out, h->x, size_t(batch) * h->cfg.d_model * 4, cudaMemcpyDeviceToDevice,
                                static_cast<cudaStream_t>(stream)));
    return DEC_OK;
}

dec_status dec_set_phase_timing(dec_handle* h, int32_t enabled) {
    if (!h) return fail(nullptr, DEC_EINVAL, "dec_set_phase_timing: null handle");
    h->phase_timing = enabled != 0;
    h->phase_n = 0;
    return DEC_OK;
}

dec_status dec_phase_times(dec_handle* h, int32_t cap, float* ms, int32_t* layer, int32_t* kind, int32_t* n) {
    if (!h || !n || (cap > 0 && (!ms || !layer || !kind))) return fail(h, DEC_EINVAL, "dec_phase_times: bad arguments");
    const int phases = h->phase_n > 0 ? static_cast<int>(h->phase_n) - 1 : 0;
    *n = phases;
    if (phases == 0) return DEC_OK;
    DEC_CUDA(h, cudaEventSynchronize(h->phase_ev[h->phase_n - 1]));
    for (int i = 0; i < phases && i < cap; ++i) {
        DEC_CUDA(h, cudaEventElapsedTime(&ms[i], h->phase_ev[i], h->phase_ev[i + 1]));
        layer[i] = h->phase_tag[i + 1][0];
        kind[i] = h->phase_tag[i + 1][1];
    }
    return DEC_OK;
}

dec_status dec_set_prefill_chunk(dec_handle* h, int32_t rows) {
    if (!h) return fail(nullptr, DEC_EINVAL, "dec_set_prefill_chunk: null handle");
    if (rows < 1 || rows > kPrefillChunk)
        return fail(h, DEC_EINVAL, "prefill chunk must be in [1, " + std::to_string(kPrefillChunk) + "]");
    h->prefill_chunk = rows;
    return DEC_OK;
}

dec_status dec_set_layer_trace(dec_handle* h, float* buf) {
    if (!h) return fail(nullptr, DEC_EINVAL, "dec_set_layer_trace: null handle");
    if (buf && (reinterpret_cast<uintptr_t>(buf) & 3)) return fail(h, DEC_EINVAL, "trace buffer must be 4-byte aligned");
    h->trace = buf;
    return DEC_OK;
}

dec_status dec_step_kernels(const dec_handle* h, int32_t* kernels) {
    if (!h || !kernels) return DEC_EINVAL;
    *kernels = h->last_step_kernels;
    return DEC_OK;
}

dec_status dec_sync(dec_handle* h, void* stream) {
    if (!h) return DEC_EINVAL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    DEC_CUDA(h, cudaStreamSynchronize(st));
    int e = 0;
    DEC_CUDA(h, cudaMemcpy(&e, h->dev_err, 4, cudaMemcpyDeviceToHost));
    if (e) h->failed = true;
    if (h->failed) return fail(h, DEC_ETIMEOUT, "a bounded device wait gave up; call dec_reset before more work");
    return DEC_OK;
}

dec_status dec_release_slot(dec_handle* h, int32_t slot) {
    if (!h) return fail(nullptr, DEC_EINVAL, "dec_release_slot: null handle");
    if (slot < 0 || slot >= h->cfg.max_slots) return fail(h, DEC_EINVAL, "slot out of range");
    shrink_slot(h, slot, 0);
    h->slot_len[slot] = 0;
    h->has_tok[slot] = 0;
    return DEC_OK;
}

dec_status dec_kv_pages_free(const dec_handle* h, int32_t* pages) {
    if (!h || !pages) return fail(nullptr, DEC_EINVAL, "dec_kv_pages_free: null pointer");
    *pages = static_cast<int32_t>(h->free_pages.size());
    return DEC_OK;
}

dec_status dec_reset(dec_handle* h) {
    if (!h) return fail(nullptr, DEC_EINVAL, "dec_reset: null handle");
    DEC_TRY(check_device(h));
    // every kernel of the handle has ended before the counters are cleared
    DEC_CUDA(h, cudaDeviceSynchronize());
    const int MB = h->max_rows, H = h->cfg.n_heads;
    for (int ci = 0; ci < h->n_chains; ++ci) {
        const Chain& ch = h->chain[ci];
        DEC_CUDA(h, cudaMemset(ch.counters, 0, size_t(MB) * H * 4));
        if (ch.mma_cnt) DEC_CUDA(h, cudaMemset(ch.mma_cnt, 0, size_t(ch.mma_cnt_len) * 4));
    }
    DEC_CUDA(h, cudaMemset(h->head_counter, 0, 16));
    DEC_CUDA(h, cudaMemset(h->keys, 0, size_t(MB) * 8));
    DEC_CUDA(h, cudaMemset(h->dev_err, 0, 4));   // the status word; the wait limit stays
    DEC_CUDA(h, cudaDeviceSynchronize());
    std::fill(h->slot_len.begin(), h->slot_len.end(), 0);
    std::fill(h->has_tok.begin(), h->has_tok.end(), 0);
    std::fill(h->has_cross.begin(), h->has_cross.end(), 0);
    for (int s2 = 0; s2 < h->cfg.max_slots; ++s2) shrink_slot(h, s2, 0);
    h->failed = false;
    return DEC_OK;
}

dec_status dec_set_wait_limit(dec_handle* h, uint64_t ns) {
    if (!h) return fail(nullptr, DEC_EINVAL, "dec_set_wait_limit: null handle");
    DEC_TRY(check_device(h));
    const unsigned long long v = ns;
    DEC_CUDA(h, cudaMemcpy(h->dev_err + 2, &v, sizeof(v), cudaMemcpyHostToDevice));
    return DEC_OK;
}

dec_status dec_debug_inject(dec_handle* h, int32_t what, int32_t value) {
    if (!h) return fail(nullptr, DEC_EINVAL, "dec_debug_inject: null handle");
    if (what != DEC_INJECT_DROP_ATTN_COPY) return fail(h, DEC_EINVAL, "dec_debug_inject: unknown injection");
    h->inject_drop = value ? 1 : 0;
    return DEC_OK;
}

void dec_debug_fail_alloc(int32_t nth) {
    g_fail_alloc_at = nth > 0 ? nth : 0;
    g_alloc_count = 0;
}

size_t dec_attention_workspace_size(int32_t batch, int32_t n_heads, int32_t ld) {
    (void)ld;
    if (batch < 1 || n_heads < 1) return 0;
    const size_t counters = ((size_t(batch) * n_heads * 4) + 255) / 256 * 256;
    return counters + size_t(batch) * n_heads * kMaxSplits * kAttnPartStride * 4;
}

dec_status dec_attention(const float* q, const float* k, const float* v, const int32_t* lens, int32_t batch,
                         int32_t n_heads, int32_t ld, int32_t tiles_per_split, float* out, void* workspace,
                         size_t workspace_bytes, void* stream) {
    auto bad = [](const char* m) { return fail(nullptr, DEC_EINVAL, std::string("dec_attention: ") + m); };
    if (!q || !k || !v || !lens || !out || !workspace) return bad("null pointer");
    if (batch < 1 || n_heads < 1 || ld < 1) return bad("batch, n_heads and ld must be >= 1");
    if (tiles_per_split < 0) return bad("tiles_per_split must be >= 0");
    if (workspace_bytes < dec_attention_workspace_size(batch, n_heads, ld)) return bad("workspace too small");
    if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(workspace)) &
        15)
        return bad("k, v and workspace must be 16-byte aligned");
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_attention, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kAttnSmemBytes));
    if (e != cudaSuccess) return cuda_fail(nullptr, e, "dec_attention: device set-up");
    const AttnLaunch p = attn_launch_plan(sms, batch * n_heads, ld, tiles_per_split);
    if (p.S > kMaxSplits) return bad("tiles_per_split gives more than 32 splits over ld rows");
    AttnArgs a{};
    a.q = q;
    a.q_bstride = (long long)n_heads * 64;
    a.k = k;
    a.v = v;
    a.slot_stride = (long long)n_heads * ld * 64;
    a.ld = ld;
    a.H = n_heads;
    a.mode = ATTN_OP;
    a.batch = batch;
    a.lens = lens;
    a.out = out;
    a.out_bstride = (long long)n_heads * 64;
    const size_t counters = ((size_t(batch) * n_heads * 4) + 255) / 256 * 256;
    a.counters = static_cast<int*>(workspace);
    a.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + counters);
    a.err = nullptr;
    a.S = p.S;
    a.tps = p.tps;
    a.stages = p.stages;
    e = launch(k_attention, dim3(a.S, n_heads, batch), dim3(kAttnThreads), attn_smem_bytes(p.stages),
               static_cast<cudaStream_t>(stream), a);
    if (e != cudaSuccess) return cuda_fail(nullptr, e, "dec_attention: k_attention launch");
    return DEC_OK;
}

dec_status dec_attention_plan(const dec_handle* h, int32_t cross, int32_t* tiles_per_split) {
    if (!h || !tiles_per_split) return fail(nullptr, DEC_EINVAL, "dec_attention_plan: null pointer");
    if (cross && h->cfg.family != DEC_FAMILY_WHISPER)
        return fail(const_cast<dec_handle*>(h), DEC_EINVAL, "dec_attention_plan: the model has no cross-attention");
    *tiles_per_split = cross ? h->tps_cross : h->tps_self;
    return DEC_OK;
}

dec_status dec_i8_dot(const int8_t* xq, const int8_t* wq, int32_t m, int32_t n, int32_t kdim, int32_t path,
                      int32_t* acc, void* stream) {
    auto bad = [](const char* msg) { return fail(nullptr, DEC_EINVAL, std::string("dec_i8_dot: ") + msg); };
    if (!xq || !wq || !acc) return bad("null pointer");
    if (m < 1 || m > 64 || n < 1 || kdim < 16 || kdim % 16) return bad("need 1 <= m <= 64, n >= 1, kdim a multiple of 16");
    if (path != DEC_I8_PATH_DP4A && path != DEC_I8_PATH_TCGEN05) return bad("unknown path");
    if ((reinterpret_cast<uintptr_t>(xq) | reinterpret_cast<uintptr_t>(wq)) & 15)
        return bad("xq and wq must be 16-byte aligned");
    dec_handle tmp;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&tmp.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(nullptr, e, "dec_i8_dot: device query");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    GemvArgs g{};
    g.xq = xq;
    g.x_ld = kdim;
    g.K = kdim;
    g.N = n;
    g.B = m;
    g.W = wq;
    g.out_i32 = acc;
    g.out_ld = n;
    if (path == DEC_I8_PATH_DP4A) {
        e = gemv_launch<int8_t, true, PRO_RAW_I8, EPI_I32, MAP_ADJ>(tmp.num_sms, g, st);
        if (e != cudaSuccess) return cuda_fail(nullptr, e, "dec_i8_dot: k_gemv launch");
        return DEC_OK;
    }
    // tcgen05: TMA maps of both operands, split-K scratch of the plan, then the same
    // kernel the decode step runs (EPI_I32 stores the exact int32 sums).
    const MmaPlan p = tc_plan(n, kdim, tmp.num_sms);
    if (!p.ok) return bad("shape not supported by the tensor-core plan");
    tmp.device = dev;
    CUtensorMap wmap, x16, x32;
    if (make_wmap(&tmp, &wmap, wq, n, kdim, false) != DEC_OK || make_wmap(&tmp, &x16, xq, m, kdim, false, 16) != DEC_OK ||
        make_wmap(&tmp, &x32, xq, m, kdim, false, 32) != DEC_OK)
        return fail(nullptr, DEC_ECUDA, "dec_i8_dot: " + tmp.err);
    const size_t pb = std::max<size_t>(16, tc_part_bytes(p, m));
    const int cl = std::max(1, tc_counters(p, m));
    void* part = nullptr;
    int* cnt = nullptr;
    float* xs = nullptr;
    e = cudaMallocAsync(&part, pb, st);
    if (e == cudaSuccess) e = cudaMallocAsync(reinterpret_cast<void**>(&cnt), size_t(cl) * 4, st);
    if (e == cudaSuccess) e = cudaMallocAsync(reinterpret_cast<void**>(&xs), size_t(m) * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(cnt, 0, size_t(cl) * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(xs, 0, size_t(m) * 4, st);
    if (e == cudaSuccess)
        e = proj_tc_launch<EPI_I32, MAP_ADJ, 1, 1>(tmp.num_sms, wmap, x16, x32, n, m, xs, part, pb, cnt, cl, g, st);
    const cudaError_t launch_err = e;
    if (part) cudaFreeAsync(part, st);
    if (cnt) cudaFreeAsync(cnt, st);
    if (xs) cudaFreeAsync(xs, st);
    if (launch_err != cudaSuccess) return cuda_fail(nullptr, launch_err, "dec_i8_dot: tcgen05 path");
    return DEC_OK;
}

}  // extern "C"
