"""Layer-local parity: every layer of the CUDA decoder against the oracle's same layer, run
from the GPU's own input residual and the GPU's own cache rows.

The GPU traces the residual leaving each layer (dec_set_layer_trace). For a sampled set of
streams, layer l of the oracle runs on the GPU's residual entering layer l and on the GPU's
K/V rows 0..n-1 of layer l (read back with dec_kv_read), so nothing accumulates across
layers: the only differences left are f32 rounding inside the one layer and, for the W8A8
model, int8 activation codes that sit on a rounding tie.

Ties. The oracle logs every activation whose x * inv lies within TIE_EPS code units of a
rounding boundary (a value the GPU's f32 arithmetic may put on the other side), and runs the
layer again with such activations rounded the other way, one tie per row per run. The sum
over runs of |alternative - oracle| is a per-element envelope: each output element may
differ from the oracle by the tolerance plus its envelope, and only elements downstream of
a tie have a non-zero envelope. Elements with no tie meet the plain tolerance.
"""
from __future__ import annotations

import copy
from collections import defaultdict
from dataclasses import dataclass, field
from typing import Callable, List, Optional

import numpy as np

import oracle
import synth
from tests._harness import ATOL, RTOL

# Code units (of the quantiser's x * 127 / amax) within which the GPU's input to the
# quantiser may fall on the other side of a rounding boundary (the oracle's NEAR_TIE_EPS).
TIE_EPS = oracle.decoder.NEAR_TIE_EPS


def _clone(st: oracle.decoder.StreamState, l: int) -> oracle.decoder.StreamState:
    """A stream state sharing every layer except l, whose K/V arrays are private copies."""
    c = copy.copy(st)
    c.k, c.v = list(st.k), list(st.v)
    c.k[l], c.v[l] = st.k[l].copy(), st.v[l].copy()
    return c


# A tighter tolerance, recorded beside the plain one: with identical inputs a correct layer
# differs from the oracle only by f32 rounding (TF32 splits and int32-to-f32 conversions
# included), far below 1e-4 relative to the residual's scale.
TIGHT_ATOL, TIGHT_RTOL = 1e-4, 1e-4


@dataclass
class Report:
    layers: int = 0
    elements: int = 0
    ties: int = 0                 # near-tie activations logged
    enveloped: int = 0            # output elements with a non-zero tie envelope
    beyond_tol: int = 0           # elements outside the plain tolerance (all explained by ties)
    max_err_no_tie: float = 0.0   # largest |gpu - oracle| where no tie reaches
    max_env: float = 0.0
    violations: List[str] = field(default_factory=list)
    tight_violations: List[str] = field(default_factory=list)

    def add(self, what, got, ref, env):
        got = np.asarray(got, np.float64)
        ref = np.asarray(ref, np.float64)
        err = np.abs(got - ref)
        tol = ATOL + RTOL * np.abs(ref)
        self.elements += err.size
        self.enveloped += int((env > 0).sum())
        self.beyond_tol += int((err > tol).sum())
        if (env == 0).any():
            self.max_err_no_tie = max(self.max_err_no_tie, float(err[env == 0].max()))
        self.max_env = max(self.max_env, float(env.max()) if env.size else 0.0)
        for lst, t in ((self.violations, tol), (self.tight_violations, TIGHT_ATOL + TIGHT_RTOL * np.abs(ref))):
            bad = err > t + env
            if bad.any():
                i = np.unravel_index(int(np.argmax(err - t - env)), err.shape)
                lst.append(f"{what}: {int(bad.sum())} of {err.size} outside tolerance + tie envelope; "
                           f"worst at {i}: gpu {got[i]!r} oracle {ref[i]!r} envelope {env[i]!r}")


class LayerLocal:
    """A GPU decoder over a workload's streams and oracle states for a sampled subset."""

    def __init__(self, wl: synth.Workload, sample: List[int], seed: int = 0,
                 oracle_weights: Optional[dict] = None, position_shift: int = 0):
        import torch
        from transformer_decoder_kv_b200 import Decoder

        self.wl, self.cfg, self.sample = wl, wl.model, list(sample)
        cfg = self.cfg
        W = synth.make_weights(cfg, seed)
        self.gpu = Decoder(cfg, W, max_slots=wl.batch, max_cache_len=wl.max_cache_len)
        self.ref = oracle.OracleDecoder(oracle_weights if oracle_weights is not None else W, wl.max_cache_len)
        self.position_shift = position_shift
        self.lens = synth.cache_lens(wl, seed).astype(np.int64)
        self.states = {}
        g = torch.Generator(device="cuda")
        for s in range(wl.batch):
            n = int(self.lens[s])
            enc = synth.encoder_hidden(cfg, s, seed) if cfg.is_whisper else None
            enc_d = torch.from_numpy(enc).cuda() if enc is not None else None
            if wl.cache_init == "prefill":
                self.gpu.prefill(s, synth.token_ids(cfg, s, n, seed), enc_d)
            else:
                if cfg.is_whisper:
                    self.gpu.prefill(s, [], enc_d)
                if s in self.sample:
                    ks, vs = zip(*(synth.seed_kv(cfg, s, l, n, seed) for l in range(cfg.n_layers)))
                    k, v = torch.from_numpy(np.stack(ks)).cuda(), torch.from_numpy(np.stack(vs)).cuda()
                else:
                    g.manual_seed(1000 + s)
                    k = torch.randn((cfg.n_layers, n, cfg.kv_dim), device="cuda", generator=g)
                    v = torch.randn((cfg.n_layers, n, cfg.kv_dim), device="cuda", generator=g)
                self.gpu.kv_append(s, 0, n, k, v)
                del k, v
            if s in self.sample:
                # the oracle's cache rows are replaced by the GPU's at every step
                self.states[s] = self.ref.new_state(enc)
        torch.cuda.synchronize()
        self.trace = torch.empty((cfg.n_layers, wl.batch, cfg.d_model), device="cuda")
        self.gpu.set_layer_trace(self.trace)

    def close(self):
        self.gpu.close()

    def _run_layer(self, l, x_in, sts, pos, flips=None, log=None):
        ref = self.ref
        clones = [_clone(st, l) for st in sts]
        ref.flips, ref.tie_log, ref.tie_eps = flips, log, TIE_EPS
        try:
            slots = [st.n for st in sts]
            x = ref.layer_forward(l, x_in, clones, slots, [p + self.position_shift for p in pos])
        finally:
            ref.flips, ref.tie_log = None, None
        k = np.stack([c.k[l][c.n] for c in clones])
        v = np.stack([c.v[l][c.n] for c in clones])
        return x, k, v

    def step(self, tokens: dict, report: Report) -> dict:
        """One decode step of every stream (tokens: stream -> token). Checks each layer of the
        sampled streams, the new K/V rows and the logits; returns the oracle's greedy pick
        for each sampled stream (computed from the GPU's final hidden state)."""
        import torch

        wl, cfg = self.wl, self.cfg
        B = wl.batch
        act = list(range(B))
        pos = [int(self.lens[s]) for s in act]
        logits = torch.empty((B, cfg.vocab), device="cuda")
        am = torch.empty(B, dtype=torch.int32, device="cuda")
        self.gpu.step(B, act, [tokens[s] for s in act], pos, pos, logits, am)
        self.gpu.sync()
        trace = self.trace.cpu().numpy()
        lg, amx = logits.cpu().numpy(), am.cpu().numpy()
        rows = [act.index(s) for s in self.sample]
        sts = [self.states[s] for s in self.sample]
        spos = [pos[r] for r in rows]
        # the GPU's cache rows 0..n of every layer (row n is this step's)
        gk, gv = [], []
        for s in self.sample:
            n = int(self.lens[s])
            k = torch.empty((cfg.n_layers, n + 1, cfg.kv_dim), device="cuda")
            v = torch.empty_like(k)
            for l in range(cfg.n_layers):
                self.gpu.kv_read(s, l, 0, n + 1, k[l], v[l])
            torch.cuda.synchronize()
            gk.append(k.cpu().numpy())
            gv.append(v.cpu().numpy())
        for i, s in enumerate(self.sample):
            st = sts[i]
            st.n = int(self.lens[s])
            for l in range(cfg.n_layers):
                st.k[l][: st.n] = gk[i][l, : st.n]
                st.v[l][: st.n] = gv[i][l, : st.n]
        x_in = self.ref.embed([tokens[s] for s in self.sample], spos)
        for l in range(cfg.n_layers):
            log = []
            own, kown, vown = self._run_layer(l, x_in, sts, spos, log=log)
            by_row = defaultdict(list)
            for site, r, c, _ in log:
                by_row[r].append((site, c))
            env = np.zeros(own.shape)
            env_k = np.zeros(kown.shape)
            env_v = np.zeros(vown.shape)
            for j in range(max((len(t) for t in by_row.values()), default=0)):
                flips = defaultdict(list)
                for r, t in by_row.items():
                    if j < len(t):
                        flips[t[j][0]].append((r, t[j][1]))
                alt, kalt, valt = self._run_layer(l, x_in, sts, spos, flips=dict(flips))
                env += np.abs(alt.astype(np.float64) - own)
                env_k += np.abs(kalt.astype(np.float64) - kown)
                env_v += np.abs(valt.astype(np.float64) - vown)
            report.layers += 1
            report.ties += len(log)
            report.add(f"layer {l} residual", trace[l][rows], own, env)
            report.add(f"layer {l} new K row", np.stack([gk[i][l, int(self.lens[s])] for i, s in enumerate(self.sample)]),
                       kown, env_k)
            report.add(f"layer {l} new V row", np.stack([gv[i][l, int(self.lens[s])] for i, s in enumerate(self.sample)]),
                       vown, env_v)
            x_in = trace[l][rows]
        # the head on the GPU's final hidden state
        ref_logits = self.ref.head(trace[cfg.n_layers - 1][rows])
        report.add("logits", lg[rows], ref_logits, np.zeros(ref_logits.shape))
        picks = {}
        for i, s in enumerate(self.sample):
            r = rows[i]
            assert int(amx[r]) == int(np.argmax(lg[r])), ("device argmax", s)
            want = oracle.argmax_first(ref_logits[i])
            if int(amx[r]) != want:
                srt = np.sort(ref_logits[i].astype(np.float64))
                margin = float(srt[-1] - srt[-2])
                if margin > 2 * (ATOL + RTOL * abs(float(srt[-1]))):
                    report.violations.append(f"stream {s}: greedy pick {int(amx[r])} vs oracle {want} "
                                             f"at top-2 margin {margin:.3g}")
            picks[s] = want
        for s in act:
            self.lens[s] += 1
        return {s: (picks[s] if s in picks else int(amx[act.index(s)])) for s in act}


def run_layer_local(wl_name: str, steps: int, sample: Optional[List[int]] = None, seed: int = 0,
                    mutate: Optional[Callable[[dict], dict]] = None, position_shift: int = 0) -> Report:
    wl = synth.workload(wl_name)
    cfg = wl.model
    lens = synth.cache_lens(wl, seed)
    if sample is None:
        order = np.argsort(lens, kind="stable")
        sample = sorted({int(order[0]), int(order[-1]), int(order[len(order) // 2])})
    ow = None
    if mutate is not None:
        ow = mutate(copy.deepcopy(synth.make_weights(cfg, seed)))
    ll = LayerLocal(wl, sample, seed, oracle_weights=ow, position_shift=position_shift)
    rep = Report()
    toks = {s: int(t) for s, t in enumerate(synth.token_ids(cfg, 4242, wl.batch, seed))}
    try:
        for _ in range(steps):
            toks = ll.step(toks, rep)
    finally:
        ll.close()
    return rep
