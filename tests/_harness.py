"""Drive the CUDA decoder (through the C ABI binding) and the CPU oracle on the same
seeded inputs, for the parity tests.

Tolerances. f32 hidden states and logits: |gpu - oracle| <= ATOL + RTOL |oracle|.
For the W8A8 models the oracle runs as a small ensemble: the oracle proper plus
N_JITTER runs that round every near-tie activation (oracle NEAR_TIE_EPS) the other way
with probability 1/2 (oracle `quant_jitter`). Each is a correct f32 implementation; they
differ where an activation sits on a rounding tie. The GPU must then lie within
ATOL + RTOL |oracle| + 2 * envelope, the envelope being the largest distance of a jittered
run from the oracle proper on that row. The strict check of the W8A8 models is the
layer-local one (tests/_layer_local.py), which needs no ensemble.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

import oracle
import synth

ATOL, RTOL = 2e-3, 1e-3
N_JITTER = 2


def within(got, ref, atol=ATOL, rtol=RTOL) -> bool:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return bool(np.all(np.abs(got - ref) <= atol + rtol * np.abs(ref)))


def close(got, ref, atol=ATOL, rtol=RTOL, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(int(np.argmax(err - bound)), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {err.size} elements outside "
                             f"atol={atol:.3g} rtol={rtol}; worst at {i}: got {got[i]!r} ref {ref[i]!r}")
    return float(err.max()) if err.size else 0.0


def top2_margin(row) -> float:
    s = np.sort(np.asarray(row, np.float64))
    return float(s[-1] - s[-2]) if len(s) > 1 else float("inf")


@dataclass
class Pair:
    """A GPU decoder and an oracle ensemble over the same streams."""
    wl: synth.Workload
    weights: dict
    gpu: object
    ref: oracle.OracleDecoder
    states: List[oracle.decoder.StreamState] = field(default_factory=list)
    lens: Optional[np.ndarray] = None
    jrefs: list = field(default_factory=list)      # [(OracleDecoder, [StreamState])]


def n_jitter(cfg) -> int:
    return N_JITTER if cfg.proj_fmt == "w8a8" else 0


def build_pair(wl: synth.Workload, seed: int = 0, streams: Optional[List[int]] = None,
               max_slots: Optional[int] = None) -> Pair:
    """Create the decoders and bring the selected streams to their initial cache state."""
    import torch
    from transformer_decoder_kv_b200 import Decoder

    cfg = wl.model
    W = synth.make_weights(cfg, seed)
    streams = list(range(wl.batch)) if streams is None else list(streams)
    gpu = Decoder(cfg, W, max_slots=max_slots or wl.batch, max_cache_len=wl.max_cache_len)
    ref = oracle.OracleDecoder(W, wl.max_cache_len)
    jrefs = [(oracle.OracleDecoder(W, wl.max_cache_len, quant_jitter=100 + j, share_weights_with=ref), [])
             for j in range(n_jitter(cfg))]
    lens_all = synth.cache_lens(wl, seed)
    p = Pair(wl, W, gpu, ref, [], lens_all[streams], jrefs)
    for slot, s in enumerate(streams):
        n = int(lens_all[s])
        enc = synth.encoder_hidden(cfg, s, seed) if cfg.is_whisper else None
        enc_d = torch.from_numpy(enc).cuda() if enc is not None else None
        if wl.cache_init == "prefill":
            toks = synth.token_ids(cfg, s, n, seed)
            gpu.prefill(slot, toks, enc_d)
            for r, sts in [(ref, p.states)] + jrefs:
                st = r.new_state(enc)
                r.prefill(st, list(toks))
                sts.append(st)
        else:
            if cfg.is_whisper:
                gpu.prefill(slot, [], enc_d)
            ks, vs = zip(*(synth.seed_kv(cfg, s, l, n, seed) for l in range(cfg.n_layers)))
            k, v = np.stack(ks), np.stack(vs)
            gpu.kv_append(slot, 0, n, torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
            for r, sts in [(ref, p.states)] + jrefs:
                st = r.new_state(enc)
                r.kv_append(st, 0, k, v)
                sts.append(st)
    torch.cuda.synchronize()
    return p


def step_refs(p: Pair, tokens, positions, idx=None):
    """Step the oracle and its jittered copies; returns (hidden, logits, env_hidden,
    env_logits) for the selected states (env = per-row largest distance of a jittered
    run from the oracle proper)."""
    idx = list(range(len(p.states))) if idx is None else idx
    rh, rl = p.ref.step([p.states[i] for i in idx], list(tokens), list(positions))
    env_h = np.zeros(len(idx))
    env_l = np.zeros(len(idx))
    for r, sts in p.jrefs:
        jh, jl = r.step([sts[i] for i in idx], list(tokens), list(positions))
        env_h = np.maximum(env_h, np.abs(jh.astype(np.float64) - rh).max(axis=1))
        env_l = np.maximum(env_l, np.abs(jl.astype(np.float64) - rl).max(axis=1))
    return rh, rl, env_h, env_l


def step_both(p: Pair, tokens, slots=None):
    """One decode step of all paired streams with the given tokens; returns
    (gpu logits, gpu argmax, gpu hidden, oracle logits, oracle hidden, env_h, env_l)."""
    import torch

    B = len(p.states)
    slots = list(range(B)) if slots is None else slots
    cfg = p.wl.model
    pos = [st.n for st in p.states]
    logits = torch.empty((B, cfg.vocab), device="cuda")
    am = torch.empty(B, dtype=torch.int32, device="cuda")
    p.gpu.step(B, slots, tokens, pos, pos, logits, am)
    hid = torch.empty((B, cfg.d_model), device="cuda")
    p.gpu.hidden(hid, B)
    p.gpu.sync()
    rh, rl, env_h, env_l = step_refs(p, tokens, pos)
    return logits.cpu().numpy(), am.cpu().numpy(), hid.cpu().numpy(), rl, rh, env_h, env_l


def check_row(gh, gl, gpick, rh, rl, env_h, env_l, what):
    """One stream's step: hidden and logits within tolerance (+ twice the ensemble
    envelope), device argmax consistent with device logits, and the greedy pick equal
    to the oracle's unless the oracle's top-2 margin is inside the tolerance."""
    close(gh, rh, atol=ATOL + 2 * env_h, what=f"{what} hidden")
    close(gl, rl, atol=ATOL + 2 * env_l, what=f"{what} logits")
    assert int(gpick) == int(np.argmax(gl)), what
    ref_pick = int(np.argmax(rl))
    if int(gpick) != ref_pick:
        m = top2_margin(rl)
        assert m <= 2 * (ATOL + 2 * env_l + RTOL * abs(float(rl[ref_pick]))), (what, m)
        return ("argmax near-tie", what, m)
    return None
