"""Drive the CUDA decoder (through the C ABI binding) and the CPU oracle on the
same seeded inputs, for the parity tests."""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

import oracle
import synth

ATOL, RTOL = 2e-3, 1e-3   # f32 hidden states and logits: |gpu - oracle| <= ATOL + RTOL |oracle|
# An int8 activation whose x * inv lies closer than this (in code units) to a rounding
# boundary k + 1/2 may round either way: two correct f32 implementations of the norm
# that feeds the quantiser differ by a few ulps, i.e. up to ~127 * 2.5e-7 = 3e-5 code
# units. 1e-4 leaves a 3x margin.
NEAR_TIE = 1e-4


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
                             f"atol={atol} rtol={rtol}; worst at {i}: got {got[i]!r} ref {ref[i]!r}")
    return float(err.max()) if err.size else 0.0


def top2_margin(row) -> float:
    s = np.sort(np.asarray(row, np.float64))
    return float(s[-1] - s[-2]) if len(s) > 1 else float("inf")


@dataclass
class Pair:
    """A GPU decoder and an oracle decoder over the same streams."""
    wl: synth.Workload
    weights: dict
    gpu: object
    ref: oracle.OracleDecoder
    states: List[oracle.decoder.StreamState] = field(default_factory=list)
    lens: Optional[np.ndarray] = None
    margins: Optional[np.ndarray] = None


def build_pair(wl: synth.Workload, seed: int = 0, streams: Optional[List[int]] = None,
               max_slots: Optional[int] = None) -> Pair:
    """Create both decoders and bring the selected streams to their initial cache state."""
    import torch
    from transformer_decoder_kv_b200 import Decoder

    cfg = wl.model
    W = synth.make_weights(cfg, seed)
    streams = list(range(wl.batch)) if streams is None else list(streams)
    gpu = Decoder(cfg, W, max_slots=max_slots or wl.batch, max_cache_len=wl.max_cache_len)
    ref = oracle.OracleDecoder(W, wl.max_cache_len)
    lens_all = synth.cache_lens(wl, seed)
    p = Pair(wl, W, gpu, ref, [], lens_all[streams])
    for slot, s in enumerate(streams):
        n = int(lens_all[s])
        enc = synth.encoder_hidden(cfg, s, seed) if cfg.is_whisper else None
        st = ref.new_state(enc)
        enc_d = torch.from_numpy(enc).cuda() if enc is not None else None
        if wl.cache_init == "prefill":
            toks = synth.token_ids(cfg, s, n, seed)
            gpu.prefill(slot, toks, enc_d)
            ref.prefill(st, list(toks))
        else:
            if cfg.is_whisper:
                gpu.prefill(slot, [], enc_d)
            ks, vs = [], []
            for l in range(cfg.n_layers):
                k, v = synth.seed_kv(cfg, s, l, n, seed)
                ks.append(k)
                vs.append(v)
            k = np.stack(ks)
            v = np.stack(vs)
            gpu.kv_append(slot, 0, n, torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
            ref.kv_append(st, 0, k, v)
        p.states.append(st)
    torch.cuda.synchronize()
    return p


def step_both(p: Pair, tokens, slots=None):
    """One decode step of all paired streams with the given tokens; returns
    (gpu logits, gpu argmax, gpu hidden, oracle logits, oracle hidden)."""
    import torch

    B = len(p.states)
    slots = list(range(B)) if slots is None else slots
    cfg = p.wl.model
    pos = [st.n for st in p.states]
    lens = [st.n for st in p.states]
    logits = torch.empty((B, cfg.vocab), device="cuda")
    am = torch.empty(B, dtype=torch.int32, device="cuda")
    p.gpu.step(B, slots, tokens, pos, lens, logits, am)
    hid = torch.empty((B, cfg.d_model), device="cuda")
    p.gpu.hidden(hid, B)
    p.gpu.sync()
    rh, rl = p.ref.step(p.states, list(tokens), pos)
    p.margins = p.ref.last_margins
    return logits.cpu().numpy(), am.cpu().numpy(), hid.cpu().numpy(), rl, rh
