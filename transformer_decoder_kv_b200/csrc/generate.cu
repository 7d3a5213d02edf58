// dec_generate: greedy generation for many requests with continuous batching, built on the
// library's own entry points (dec_prefill, dec_step, dec_next_tokens).
//
// franken_ocr decoder_qwen2.rs, `BatchScheduler::run` / `generate_greedy_batched`: requests
// wait in arrival order; whenever a slot is free the next request is admitted (its prompt is
// prefilled and the prompt's last-row argmax is its first token); every iteration advances
// all admitted streams by one token with a single batched decode step; a stream retires when
// it emits its stop token or reaches its own token cap, and its slot is backfilled from the
// queue before the next step. Each stream's tokens depend only on its own request: the step's
// per-stream arithmetic does not depend on the rest of the batch (W8A8 and the head exactly;
// attention splits by each row's own length), which the tests check against solo runs.

#include <algorithm>
#include <deque>
#include <string>
#include <vector>

#include "../../include/dec.h"

void dec_set_thread_error(const char* msg);

namespace {

struct Stream {
    int req;
    int slot;
    int emitted;   // tokens written to the request's output
    int len;       // cached rows of the slot
    int last;      // last emitted token
    int pages;     // cache pages reserved for the stream (paged cache)
};

dec_status gen_fail(dec_status st, const std::string& msg) {
    dec_set_thread_error(("dec_generate: " + msg).c_str());
    return st;
}

}  // namespace

extern "C" dec_status dec_generate(dec_handle* h, const dec_request* reqs, int32_t n_reqs, int32_t max_active,
                                   int32_t* tokens_out, int32_t stride, int32_t* n_out, void* stream) {
    if (!h) return gen_fail(DEC_EINVAL, "null handle");
    if (n_reqs < 0 || (n_reqs > 0 && (!reqs || !tokens_out || !n_out))) return gen_fail(DEC_EINVAL, "bad arguments");
    if (max_active < 1) return gen_fail(DEC_EINVAL, "max_active must be >= 1");
    dec_config c;
    dec_status st = dec_get_config(h, &c);
    if (st != DEC_OK) return st;
    const bool whisper = c.family == DEC_FAMILY_WHISPER;
    for (int r = 0; r < n_reqs; ++r) {
        const dec_request& q = reqs[r];
        const std::string who = "request " + std::to_string(r) + ": ";
        if (!q.prompt || q.n_prompt < 1) return gen_fail(DEC_EINVAL, who + "needs a prompt of at least one token");
        if (q.n_prompt > c.max_cache_len) return gen_fail(DEC_EOVERFLOW, who + "prompt longer than max_cache_len");
        if (q.n_prompt > c.max_pos) return gen_fail(DEC_ERANGE, who + "prompt longer than the position range");
        if (q.max_new < 1 || q.max_new > stride) return gen_fail(DEC_EINVAL, who + "max_new must be in [1, stride]");
        if (q.eos < -1 || q.eos >= c.vocab) return gen_fail(DEC_ERANGE, who + "eos outside [-1, vocab)");
        if (whisper != (q.enc_hidden != nullptr))
            return gen_fail(DEC_EINVAL, who + (whisper ? "whisper needs enc_hidden" : "enc_hidden must be NULL"));
        for (int i = 0; i < q.n_prompt; ++i)
            if (q.prompt[i] < 0 || q.prompt[i] >= c.vocab) return gen_fail(DEC_ERANGE, who + "prompt token outside vocab");
    }
    // A paged cache admits a request only while the pages of its longest possible stream
    // (prompt + max_new rows, at most max_cache_len) fit next to those reserved by the
    // streams already running, so no running stream can find the pool empty.
    const int P = c.kv_page_rows;
    auto pages_for = [&](int r) {
        return P > 0 ? (std::min(reqs[r].n_prompt + reqs[r].max_new, c.max_cache_len) + P - 1) / P : 0;
    };
    for (int r = 0; r < n_reqs; ++r)
        if (pages_for(r) > c.kv_pages && P > 0)
            return gen_fail(DEC_ENOMEM, "request " + std::to_string(r) + " needs more cache pages than the pool has");
    int reserved = 0;
    const int cap = std::min(std::min(max_active, c.max_slots), DEC_MAX_BATCH);
    std::vector<int> free_slots;
    for (int s = cap - 1; s >= 0; --s) free_slots.push_back(s);   // slot 0 is taken first
    std::deque<int> pending;
    for (int r = 0; r < n_reqs; ++r) {
        pending.push_back(r);
        n_out[r] = 0;
    }
    // a stream is done once it emitted its stop token or its cap, or when its next step
    // would overflow the cache or run past the position range
    auto done = [&](const Stream& a) {
        const dec_request& q = reqs[a.req];
        return a.last == q.eos || a.emitted >= q.max_new || a.len + 1 > c.max_cache_len || a.len >= c.max_pos;
    };
    auto emit = [&](Stream& a, int tok) {
        tokens_out[static_cast<long long>(a.req) * stride + a.emitted] = tok;
        a.emitted += 1;
        a.last = tok;
        n_out[a.req] = a.emitted;
    };
    std::vector<Stream> act;
    std::vector<int32_t> slots, pos, toks;
    while (true) {
        // admit waiting requests into free slots
        while (!free_slots.empty() && !pending.empty() &&
               (P == 0 || reserved + pages_for(pending.front()) <= c.kv_pages)) {
            const int r = pending.front();
            pending.pop_front();
            Stream a{r, free_slots.back(), 0, reqs[r].n_prompt, -1, pages_for(r)};
            free_slots.pop_back();
            reserved += a.pages;
            st = dec_prefill(h, a.slot, reqs[r].prompt, reqs[r].n_prompt, reqs[r].enc_hidden, nullptr, stream);
            if (st != DEC_OK) return st;
            int32_t first = 0;
            st = dec_next_tokens(h, 1, &a.slot, &first, stream);
            if (st != DEC_OK) return st;
            emit(a, first);
            if (done(a)) {
                st = dec_release_slot(h, a.slot);
                if (st != DEC_OK) return st;
                free_slots.push_back(a.slot);
                reserved -= a.pages;
            } else {
                act.push_back(a);
            }
        }
        if (act.empty()) {
            if (pending.empty()) break;
            continue;
        }
        // one decode step over every admitted stream; each feeds its own previous pick
        const int B = static_cast<int>(act.size());
        slots.resize(B);
        pos.resize(B);
        toks.resize(B);
        for (int i = 0; i < B; ++i) {
            slots[i] = act[i].slot;
            pos[i] = act[i].len;
        }
        st = dec_step(h, B, slots.data(), nullptr, pos.data(), pos.data(), nullptr, nullptr, stream);
        if (st != DEC_OK) return st;
        st = dec_next_tokens(h, B, slots.data(), toks.data(), stream);
        if (st != DEC_OK) return st;
        std::vector<Stream> keep;
        keep.reserve(act.size());
        for (int i = 0; i < B; ++i) {
            Stream& a = act[i];
            a.len += 1;
            emit(a, toks[i]);
            if (done(a)) {
                st = dec_release_slot(h, a.slot);
                if (st != DEC_OK) return st;
                free_slots.push_back(a.slot);
                reserved -= a.pages;
            } else {
                keep.push_back(a);
            }
        }
        act.swap(keep);
    }
    return DEC_OK;
}
