"""Continuous batching (dec_generate) and free-running greedy sequences.

* Batched equals solo: the token ids of every request are the same when the requests are
  run one at a time and when up to 9 run together with admission, retirement at a stop token
  or at per-request caps, and backfill from the queue (franken_ocr decoder_qwen2.rs tests:
  batched ids equal solo ids with mixed caps and mid-stream EOS).
* Greedy sequences identical to the oracle's, free-running (each side feeds its own picks):
  small models, the C3 workload (1024-token prompt, then 128 greedy steps), one sampled C5
  stream (4-token prompt, 200 steps) while all 32 run, and sampled C4 streams over 32 steps.
  Where the oracle's top-2 margin at a step is inside the logit tolerance the two may pick
  differently; such a step is reported and ends the comparison of that stream.
"""
import numpy as np
import pytest

import oracle
import synth
from tests._harness import ATOL, RTOL

pytestmark = pytest.mark.gpu


def _margin(row):
    s = np.sort(np.asarray(row, np.float64))
    return float(s[-1] - s[-2]), float(s[-1])


def oracle_greedy(ref, prompt, max_new, eos=-1, enc=None, max_len=None, max_pos=None):
    """The oracle's greedy generation: prefill, then one step per token; returns the ids and
    each pick's (top-2 margin, top value)."""
    st = ref.new_state(enc)
    logits = ref.prefill(st, list(prompt))
    ids, margins = [], []
    while True:
        tok = oracle.argmax_first(logits)
        ids.append(tok)
        margins.append(_margin(logits))
        if tok == eos or len(ids) >= max_new or st.n + 1 > (max_len or ref.max_len) or \
                (max_pos is not None and st.n >= max_pos):
            return ids, margins
        _, lg = ref.step([st], [tok], [st.n])
        logits = lg[0]


def compare_greedy(gpu_ids, ref_ids, margins, what, env_at=None):
    """Identical sequences, or a divergence at a near-tie (reported); returns the event.

    A near-tie is a top-2 margin inside twice the logit tolerance. For the W8A8 models
    `env_at(i)` gives the spread of the oracle ensemble (tests/_harness.py) at pick i with the
    same history: correct implementations whose int8 activation codes round differently at
    ties drift apart by that much over the layers, so a margin inside twice the tolerance plus
    that spread is a near-tie too."""
    for i, (g, o) in enumerate(zip(gpu_ids, ref_ids)):
        if g != o:
            m, top = margins[i]
            env = env_at(i) if env_at is not None else 0.0
            assert m <= 2 * (ATOL + RTOL * abs(top) + 2 * env), (what, i, g, o, m, env)
            return (what, "near-tie divergence at token", i, m, env)
    assert len(gpu_ids) == len(ref_ids), (what, len(gpu_ids), len(ref_ids))
    return None


def ensemble_env(W, max_len, start, tokens, n_jitter=2):
    """Largest distance of a jittered oracle's logits from the oracle proper's after `start`
    (a function giving a fresh decoder's stream state and first logits) and the teacher-forced
    `tokens` (the same history for all)."""
    runs = []
    for seed in [None] + [100 + j for j in range(n_jitter)]:
        r = oracle.OracleDecoder(W, max_len, quant_jitter=seed)
        st, lg = start(r)
        for t in tokens:
            _, l = r.step([st], [t], [st.n])
            lg = l[0]
        runs.append(np.asarray(lg, np.float64))
    return max(float(np.abs(j - runs[0]).max()) for j in runs[1:])


def _requests(cfg, n, seed=0):
    import torch
    r = np.random.default_rng(seed)
    reqs = []
    for i in range(n):
        plen = int(r.integers(1, 24))
        req = {"prompt": [int(t) for t in synth.token_ids(cfg, 500 + i, plen, seed)],
               "max_new": int(r.integers(1, 18))}
        if cfg.is_whisper:
            req["enc_hidden"] = torch.from_numpy(synth.encoder_hidden(cfg, i, seed)).cuda()
        reqs.append(req)
    return reqs


@pytest.mark.parametrize("name,max_active", [("mid_qwen2", 9), ("tiny_qwen2", 5), ("tiny_whisper", 6)])
def test_generate_batched_equals_solo_with_stops_and_caps(name, max_active):
    from transformer_decoder_kv_b200 import Decoder

    cfg = synth.MODELS[name]
    W = synth.make_weights(cfg, 0)
    dec = Decoder(cfg, W, max_slots=max_active, max_cache_len=64)
    reqs = _requests(cfg, 14)
    free = dec.generate(reqs, max_active=1)
    # mid-stream stops: a request stops at the token its free run emitted at some step
    r = np.random.default_rng(1)
    for i, ids in enumerate(free):
        if len(ids) > 2 and i % 3 == 0:
            reqs[i]["eos"] = ids[int(r.integers(1, len(ids) - 1))]
    solo = dec.generate(reqs, max_active=1)
    batched = dec.generate(reqs, max_active=max_active)
    assert batched == solo
    for i, ids in enumerate(solo):
        assert 1 <= len(ids) <= reqs[i]["max_new"]
        if reqs[i].get("eos", -1) >= 0:
            assert ids[-1] == reqs[i]["eos"] and reqs[i]["eos"] not in ids[:-1]
    dec.close()


@pytest.mark.parametrize("name", ["tiny_qwen2", "tiny_whisper", "tiny_whisper_w8a32"])
def test_generate_matches_oracle_greedy(name):
    from transformer_decoder_kv_b200 import Decoder

    cfg = synth.MODELS[name]
    W = synth.make_weights(cfg, 0)
    dec = Decoder(cfg, W, max_slots=4, max_cache_len=64)
    ref = oracle.OracleDecoder(W, 64)
    reqs = _requests(cfg, 4, seed=3)
    for q in reqs:
        q["max_new"] = 20
    got = dec.generate(reqs, max_active=4)
    events = []
    for i, q in enumerate(reqs):
        enc = q["enc_hidden"].cpu().numpy() if cfg.is_whisper else None
        ids, margins = oracle_greedy(ref, q["prompt"], q["max_new"], enc=enc, max_pos=cfg.max_pos)
        ev = compare_greedy(got[i], ids, margins, f"{name} request {i}")
        if ev:
            events.append(ev)
    print(events)
    dec.close()


def test_c3_prefill_1024_then_128_greedy_steps_match_oracle():
    """The C3 workload end to end: a 1024-token prompt, then 128 greedy steps (129 tokens,
    the first from the prompt's last row), free-running on both sides."""
    from transformer_decoder_kv_b200 import Decoder

    wl = synth.workload("c3_qwen2_0_5b_int8_b1")
    cfg = wl.model
    W = synth.make_weights(cfg, 0)
    dec = Decoder(cfg, W, max_slots=1, max_cache_len=wl.max_cache_len)
    n = int(synth.cache_lens(wl, 0)[0])
    prompt = [int(t) for t in synth.token_ids(cfg, 0, n, 0)]
    got = dec.generate([{"prompt": prompt, "max_new": wl.steps + 1}], max_active=1)[0]
    dec.close()
    ref = oracle.OracleDecoder(W, wl.max_cache_len)
    ids, margins = oracle_greedy(ref, prompt, wl.steps + 1)

    def start(r):
        st = r.new_state(None)
        return st, r.prefill(st, prompt)

    env_at = lambda i: ensemble_env(W, wl.max_cache_len, start, ids[:i])
    print(compare_greedy(got, ids, margins, "c3", env_at), f"min margin {min(m for m, _ in margins):.4g}")


def test_c5_sampled_stream_200_greedy_steps_match_oracle():
    """C5: all 32 streams generate (4-token prompts, 200 greedy steps after the prompt) in
    one continuous batch; stream 0 is followed by the oracle."""
    import torch
    from transformer_decoder_kv_b200 import Decoder

    wl = synth.workload("c5_whisper_large_v3_w8a32_b32")
    cfg = wl.model
    W = synth.make_weights(cfg, 0)
    dec = Decoder(cfg, W, max_slots=wl.batch, max_cache_len=wl.max_cache_len)
    lens = synth.cache_lens(wl, 0)
    reqs = []
    for s in range(wl.batch):
        reqs.append({"prompt": [int(t) for t in synth.token_ids(cfg, s, int(lens[s]), 0)],
                     "max_new": wl.steps + 1,
                     "enc_hidden": torch.from_numpy(synth.encoder_hidden(cfg, s, 0)).cuda()})
    got = dec.generate(reqs, max_active=wl.batch)
    dec.close()
    assert all(len(g) == wl.steps + 1 for g in got)
    ref = oracle.OracleDecoder(W, wl.max_cache_len)
    del W
    ids, margins = oracle_greedy(ref, reqs[0]["prompt"], wl.steps + 1, enc=synth.encoder_hidden(cfg, 0, 0),
                                 max_pos=cfg.max_pos)
    print(compare_greedy(got[0], ids, margins, "c5 stream 0"), f"min margin {min(m for m, _ in margins):.4g}")


def test_c4_sampled_streams_32_greedy_steps_match_oracle():
    """C4: 64 streams over seeded caches step 32 times feeding their own picks (tokens =
    NULL); the shortest and the longest stream are followed by the oracle."""
    import torch
    from transformer_decoder_kv_b200 import Decoder

    wl = synth.workload("c4_qwen2_0_5b_int8_b64")
    cfg = wl.model
    W = synth.make_weights(cfg, 0)
    dec = Decoder(cfg, W, max_slots=wl.batch, max_cache_len=wl.max_cache_len)
    ref = oracle.OracleDecoder(W, wl.max_cache_len)
    lens = synth.cache_lens(wl, 0).astype(np.int64)
    sample = sorted({int(np.argmin(lens)), int(np.argmax(lens))})
    states = {}
    g = torch.Generator(device="cuda")
    for s in range(wl.batch):
        n = int(lens[s])
        if s in sample:
            ks, vs = zip(*(synth.seed_kv(cfg, s, l, n, 0) for l in range(cfg.n_layers)))
            k, v = np.stack(ks), np.stack(vs)
            dec.kv_append(s, 0, n, torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
            st = ref.new_state(None)
            ref.kv_append(st, 0, k, v)
            states[s] = st
        else:
            g.manual_seed(1000 + s)
            dec.kv_append(s, 0, n, torch.randn((cfg.n_layers, n, cfg.kv_dim), device="cuda", generator=g),
                          torch.randn((cfg.n_layers, n, cfg.kv_dim), device="cuda", generator=g))
    first = [int(t) for t in synth.token_ids(cfg, 4242, wl.batch, 0)]
    am = torch.empty(wl.batch, dtype=torch.int32, device="cuda")
    gpu_ids = {s: [] for s in sample}
    for t in range(wl.steps):
        pos = [int(x) for x in lens]
        dec.step(wl.batch, None, first if t == 0 else None, pos, pos, None, am)
        picks = am.cpu().numpy()
        for s in sample:
            gpu_ids[s].append(int(picks[s]))
        lens += 1
    dec.close()
    for s in sample:
        st = states[s]
        tok, ids, margins = first[s], [], []
        for t in range(wl.steps):
            _, lg = ref.step([st], [tok], [st.n])
            tok = oracle.argmax_first(lg[0])
            ids.append(tok)
            margins.append(_margin(lg[0]))
        n0 = int(synth.cache_lens(wl, 0)[s])

        def start(r, s=s, n0=n0):
            ks, vs = zip(*(synth.seed_kv(cfg, s, l, n0, 0) for l in range(cfg.n_layers)))
            st2 = r.new_state(None)
            r.kv_append(st2, 0, np.stack(ks), np.stack(vs))
            _, lg0 = r.step([st2], [first[s]], [st2.n])
            return st2, lg0[0]

        env_at = lambda i, start=start, ids=ids: ensemble_env(W, wl.max_cache_len, start, ids[:i])
        print(compare_greedy(gpu_ids[s], ids, margins, f"c4 stream {s}", env_at),
              f"min margin {min(m for m, _ in margins):.4g}")
