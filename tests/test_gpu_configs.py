"""Full-size parity: the five decode workloads at their real shapes and batch sizes.

The GPU runs every stream of the batch, in the launch configuration the benchmark
times. The oracle follows a few sampled streams (streams are independent, so a
sampled stream's results do not depend on the others): the shortest, the longest
and one in between. Steps are teacher-forced: sampled streams receive the oracle's
greedy pick, the others their own device pick. For the W8A8 model the oracle runs
as an ensemble with jittered quantiser inputs (see tests/_harness.py).
"""
import numpy as np
import pytest

import oracle
import synth
from tests._harness import check_row, n_jitter

pytestmark = pytest.mark.gpu


def _sample(lens, k=3):
    order = np.argsort(lens, kind="stable")
    pick = [int(order[0]), int(order[-1]), int(order[len(order) // 2])]
    return sorted(set(pick))[:k]


def _setup(wl, sample, seed=0):
    import torch
    from transformer_decoder_kv_b200 import Decoder

    cfg = wl.model
    W = synth.make_weights(cfg, seed)
    gpu = Decoder(cfg, W, max_slots=wl.batch, max_cache_len=wl.max_cache_len)
    ref = oracle.OracleDecoder(W, wl.max_cache_len)
    refs = [ref] + [oracle.OracleDecoder(W, wl.max_cache_len, quant_jitter=100 + j, share_weights_with=ref)
                    for j in range(n_jitter(cfg))]
    del W
    lens = synth.cache_lens(wl, seed)
    states = [dict() for _ in refs]
    g = torch.Generator(device="cuda")
    for s in range(wl.batch):
        n = int(lens[s])
        enc = synth.encoder_hidden(cfg, s, seed) if cfg.is_whisper else None
        enc_d = torch.from_numpy(enc).cuda() if enc is not None else None
        if wl.cache_init == "prefill":
            toks = synth.token_ids(cfg, s, n, seed)
            gpu.prefill(s, toks, enc_d)
            if s in sample:
                for r, sts in zip(refs, states):
                    st = r.new_state(enc)
                    r.prefill(st, list(toks))
                    sts[s] = st
        else:
            if cfg.is_whisper:
                gpu.prefill(s, [], enc_d)
            if s in sample:
                ks, vs = zip(*(synth.seed_kv(cfg, s, l, n, seed) for l in range(cfg.n_layers)))
                k, v = np.stack(ks), np.stack(vs)
                gpu.kv_append(s, 0, n, torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
                for r, sts in zip(refs, states):
                    st = r.new_state(enc)
                    r.kv_append(st, 0, k, v)
                    sts[s] = st
            else:
                g.manual_seed(1000 + s)
                k = torch.randn((cfg.n_layers, n, cfg.kv_dim), device="cuda", generator=g)
                v = torch.randn((cfg.n_layers, n, cfg.kv_dim), device="cuda", generator=g)
                gpu.kv_append(s, 0, n, k, v)
                del k, v
    torch.cuda.synchronize()
    return gpu, refs, states, lens.astype(np.int64)


def _run_config(wl_name, steps, seed=0):
    import torch

    wl = synth.workload(wl_name)
    cfg = wl.model
    lens0 = synth.cache_lens(wl, seed)
    sample = _sample(lens0)
    gpu, refs, states, lens = _setup(wl, sample, seed)
    B = wl.batch
    limit = wl.retire_at or wl.max_cache_len
    toks = {s: int(t) for s, t in enumerate(synth.token_ids(cfg, 4242, B, seed))}
    events = []
    logits = torch.empty((B, cfg.vocab), device="cuda")
    am = torch.empty(B, dtype=torch.int32, device="cuda")
    hid = torch.empty((B, cfg.d_model), device="cuda")
    for t in range(steps):
        act = [s for s in range(B) if lens[s] < limit and lens[s] + 1 <= wl.max_cache_len]
        if not act:
            break
        pos = [int(lens[s]) for s in act]
        gpu.step(len(act), act, [toks[s] for s in act], pos, pos, logits, am)
        gpu.hidden(hid, len(act))
        gpu.sync()
        lg = logits[: len(act)].cpu().numpy()
        ams = am[: len(act)].cpu().numpy()
        hd = hid[: len(act)].cpu().numpy()
        ref_act = [s for s in act if s in states[0]]
        outs = [r.step([sts[s] for s in ref_act], [toks[s] for s in ref_act], [int(lens[s]) for s in ref_act])
                for r, sts in zip(refs, states)]
        rh, rl = outs[0]
        env_h = np.zeros(len(ref_act))
        env_l = np.zeros(len(ref_act))
        for jh, jl in outs[1:]:
            env_h = np.maximum(env_h, np.abs(jh.astype(np.float64) - rh).max(axis=1))
            env_l = np.maximum(env_l, np.abs(jl.astype(np.float64) - rl).max(axis=1))
        for i, s in enumerate(act):
            assert np.all(np.isfinite(lg[i])), (t, s)
            assert int(ams[i]) == int(np.argmax(lg[i])), (t, s)
        for j, s in enumerate(ref_act):
            i = act.index(s)
            ev = check_row(hd[i], lg[i], ams[i], rh[j], rl[j], env_h[j], env_l[j],
                           f"{wl_name} step {t} stream {s}")
            if ev:
                events.append(ev)
            if env_l[j] > 0:
                events.append(("ensemble envelope", t, s, float(env_l[j])))
        for i, s in enumerate(act):
            lens[s] += 1
            toks[s] = int(np.argmax(rl[ref_act.index(s)])) if s in states[0] else int(ams[i])
    gpu.close()
    if events:
        print(f"{wl_name}: {events}")
    return events


def test_c1_whisper_tiny_block_b1():
    _run_config("c1_whisper_tiny_block_b1", steps=4)


def test_c2_whisper_base_b16():
    _run_config("c2_whisper_base_b16", steps=4)


def test_c3_qwen2_0_5b_int8_b1():
    _run_config("c3_qwen2_0_5b_int8_b1", steps=4)


def test_c4_qwen2_0_5b_int8_b64():
    _run_config("c4_qwen2_0_5b_int8_b64", steps=3)


def test_c5_whisper_large_v3_w8a32_b32():
    _run_config("c5_whisper_large_v3_w8a32_b32", steps=3)
