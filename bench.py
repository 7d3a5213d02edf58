"""Benchmark of the batched single-token decode step on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--config c4] [--impl ours|reference]

Prints ONE JSON line (rank 0). `value` is decode tokens/s over all ranks, device-
timed with CUDA events around K consecutive dec_step calls (greedy continuation on
the device, no host round trip), max over ranks. `e2e` is the same metric through
dec_step_host (host token/position/length arrays in, host logits and argmax out,
synchronised every step). `roofline` reports the dominant kernel of the workload
timed on its own with CUDA events against the measured HBM copy bandwidth.
`cpu_baseline` times the CPU oracle on a bounded sample of the same workload.
Streams are independent, so N ranks run N independent replicas (weak scaling,
no collective on the data path).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

CONFIGS = {
    "c1": "c1_whisper_tiny_block_b1",
    "c2": "c2_whisper_base_b16",
    "c3": "c3_qwen2_0_5b_int8_b1",
    "c4": "c4_qwen2_0_5b_int8_b64",
    "c5": "c5_whisper_large_v3_w8a32_b32",
}
L2_BYTES = 126 * 1024 * 1024
SPLIT_MIN_BATCH = 16   # decode steps of this many rows run as several chains (the library's rule)
MAX_CHAINS = 2


def chain_rows(B: int):
    """Chain count and rows of the first chain of a split step (the library's chain_bounds)."""
    n = max(1, min(MAX_CHAINS, B // 8))
    base = max(1, (B // n) // 8 * 8)
    return n, base


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------- algorithmic bytes

def step_bytes(cfg: synth.ModelConfig, lens, head: str = "exact") -> dict:
    """Bytes one decode step must move (each weight once, caches read, rows written). The
    head is the f32 embedding (V d 4 bytes), or for the int8 head its int8 rows and row
    scales (V d + 4 V bytes; the candidates' exact re-score is a few rows)."""
    d, F, L, V = cfg.d_model, cfg.d_ff, cfg.n_layers, cfg.vocab
    B = len(lens)
    wb = 4 if cfg.proj_fmt == "f32" else 1
    if cfg.is_whisper:
        nW = L * (4 * d * d + 2 * d * d + 2 * d * F)      # q,k,v,o, xq,xo, fc1,fc2
        rows = L * (6 * d + F + d)
        small = L * (3 * 2 * d) * 4                         # three LayerNorms
    else:
        nW = L * (2 * d * d + 2 * cfg.kv_dim * d + 3 * d * F)
        rows = L * (2 * d + 2 * cfg.kv_dim + 2 * F + d)
        small = L * (2 * d) * 4
    weights = nW * wb + (rows * 4 if wb == 1 else 0) + rows * 4 * (1 if cfg.is_whisper else 0) + small
    if not cfg.is_whisper:
        weights += L * (d + 2 * cfg.kv_dim) * 4             # q/k/v biases
    head = V * d * 4 if head == "exact" else V * d + V * 4
    kvd = cfg.kv_dim
    self_kv = sum(L * (int(n) + 1) * kvd * 2 * 4 for n in lens)
    kv_write = B * L * kvd * 2 * 4
    cross = B * L * cfg.enc_len * d * 2 * 4 if cfg.is_whisper else 0
    logits = B * V * 4
    emb = B * d * 4 * (2 if cfg.is_whisper else 1)
    total = weights + head + self_kv + kv_write + cross + logits + emb
    return dict(weights=weights, head=head, self_kv=self_kv, cross=cross, total=total)


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        # samples go to a scratch file; the summary is part of the JSON line
        self.path = os.path.join(tempfile.gettempdir(), f"dec_bench_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def clocks_rejected(clocks: dict) -> bool:
    """A timed region whose clock record shows a hardware or thermal slowdown, or SM clocks
    held well below their maximum with no reason given (a leftover clock lock), does not
    give a valid number; power capping alone is kept (normal on a 1 kW part)."""
    reasons = set(clocks.get("reasons") or [])
    if reasons & {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}:
        return True
    sm, smax = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if sm and smax and sm < 0.8 * smax and not (reasons & {"sw_power_cap"}):
        return True
    return False


# ---------------------------------------------------------------- workload setup (GPU)

class GpuWorkload:
    """The workload's decoder with its streams brought to their initial cache state."""

    def __init__(self, wl: synth.Workload, seed: int, fast_setup: bool = False, head: str = "exact"):
        import torch
        from transformer_decoder_kv_b200 import Decoder

        self.wl = wl
        cfg = wl.model
        self.cfg = cfg
        W = synth.make_weights(cfg, seed)
        self.dec = Decoder(cfg, W, max_slots=wl.batch, max_cache_len=wl.max_cache_len, head=head)
        del W
        self.lens0 = synth.cache_lens(wl, seed).astype(np.int64)
        B = wl.batch
        if wl.cache_init == "prefill" and not fast_setup:
            for s in range(B):
                enc = torch.from_numpy(synth.encoder_hidden(cfg, s, seed)).cuda() if cfg.is_whisper else None
                self.dec.prefill(s, synth.token_ids(cfg, s, int(self.lens0[s]), seed), enc)
        else:
            # seeded N(0,1) K/V rows (profiling shortcut for prefill workloads: same
            # shapes and lengths, so the same decode-step cost)
            g = torch.Generator(device="cuda")
            for s in range(B):
                n = int(self.lens0[s])
                if cfg.is_whisper:
                    enc = torch.from_numpy(synth.encoder_hidden(cfg, s, seed)).cuda()
                    self.dec.prefill(s, [], enc)
                g.manual_seed(seed * 100003 + s)
                k = torch.randn((cfg.n_layers, n, cfg.kv_dim), device="cuda", generator=g)
                v = torch.randn((cfg.n_layers, n, cfg.kv_dim), device="cuda", generator=g)
                self.dec.kv_append(s, 0, n, k, v)
                del k, v
        # the first step feeds one seeded token per stream; later steps continue greedily
        self.first_tokens = synth.token_ids(cfg, 7777, B, seed)
        torch.cuda.synchronize()
        self.lens = self.lens0.copy()
        self.started = wl.cache_init == "prefill" and not fast_setup
        self.t = 0
        self.logits = torch.empty((B, cfg.vocab), device="cuda")
        self.argmax = torch.empty(B, dtype=torch.int32, device="cuda")

    def _plan(self):
        """Streams active at the next step (retired ones leave the batch). After the
        workload's step count the caches are rewound to their initial lengths."""
        wl = self.wl
        if self.t >= wl.steps:
            for s in range(wl.batch):
                self.dec.kv_append(s, int(self.lens0[s]), 0, None, None)
            self.lens = self.lens0.copy()
            self.t = 0
        lim = wl.retire_at if wl.retire_at else wl.max_cache_len
        act = [s for s in range(wl.batch) if self.lens[s] < lim and self.lens[s] + 1 <= wl.max_cache_len]
        return act

    def step(self, stream: int):
        act = self._plan()
        B = len(act)
        pos = [int(self.lens[s]) for s in act]
        toks = None  # greedy continuation on the device
        if not self.started:
            toks = [int(self.first_tokens[s]) for s in act]
            self.started = True
        self.dec.step(B, act, toks, pos, pos, self.logits, self.argmax, stream)
        for s in act:
            self.lens[s] += 1
        self.t += 1
        return B, pos


def run_ours(args, wl: synth.Workload, rank: int, world: int) -> dict:
    import torch

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
    seed = rank
    cfg = wl.model
    gw = GpuWorkload(wl, seed, fast_setup=args.fast_setup, head=args.head)
    stream = torch.cuda.Stream()
    sh = stream.cuda_stream
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            gw.step(sh)
        torch.cuda.synchronize()
        lens_at_start = gw.lens.copy()
        t_at_start = gw.t
        _barrier(world)
        clk = ClockSampler(torch.cuda.current_device())
        clk.start()
        time.sleep(0.3)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        tokens = 0
        lens_seen = []
        launches = 0
        if args.profile_range:
            torch.cuda.profiler.start()
        e0.record(stream)
        for _ in range(args.steps):
            b, pos = gw.step(sh)
            tokens += b
            lens_seen.append(pos)
            launches += gw.dec.step_kernels()
        e1.record(stream)
        torch.cuda.synchronize()
        if args.profile_range:
            torch.cuda.profiler.stop()
        clocks = clk.stop()
        clocks["rejected"] = clocks_rejected(clocks)
        ms = e0.elapsed_time(e1)
        gw.dec.sync(sh)
    value, ms_max, tokens_all = combine_ranks(ms, tokens, world)

    # bytes actually moved per step at the lengths seen
    per_step_bytes = [step_bytes(cfg, p, args.head)["total"] for p in lens_seen]
    achieved_gbs = sum(per_step_bytes) / (ms / 1e3) / 1e9

    # ---- e2e through host buffers ----
    with torch.cuda.stream(stream):
        Bmax = wl.batch
        lh = torch.empty((Bmax, cfg.vocab), dtype=torch.float32).pin_memory().numpy()
        ah = torch.zeros(Bmax, dtype=torch.int32).pin_memory().numpy()
        # the host path feeds its own previous picks back as host tokens
        ah[:] = 0
        gw.started = True
        ee0 = torch.cuda.Event(enable_timing=True)
        ee1 = torch.cuda.Event(enable_timing=True)
        e2e_tokens = 0
        e2e_steps = max(1, min(args.steps, 32))
        torch.cuda.synchronize()
        ee0.record(stream)
        for _ in range(e2e_steps):
            act = gw._plan()
            B = len(act)
            pos = [int(gw.lens[s]) for s in act]
            toks = [int(x) for x in ah[:B]]
            gw.dec.step_host(B, act, toks, pos, pos, lh[:B], ah[:B], sh)
            for s in act:
                gw.lens[s] += 1
            gw.t += 1
            e2e_tokens += B
        ee1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = ee0.elapsed_time(ee1)
    e2e_value = combine_ranks(e2e_ms, e2e_tokens, world)[0]
    meta_bytes = 4 * 4 * wl.batch  # slots, tokens, positions, lengths
    e2e = {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": meta_bytes,
           "d2h_bytes_per_step": wl.batch * (cfg.vocab * 4 + 4)}

    tps = gw.dec.attention_plan(cross=cfg.is_whisper)
    roof = dominant_kernel_roofline(wl, cfg, lens_at_start, tps) if rank == 0 else None
    gw.dec.close()
    return dict(value=value, ms=ms_max, tokens=tokens_all, clocks=clocks, e2e=e2e, roofline=roof,
                achieved_gbs=achieved_gbs, launches=launches,
                step_bytes=statistics.mean(per_step_bytes))


def dominant_kernel_roofline(wl, cfg, lens, tiles_per_split: int) -> dict:
    """Time the workload's dominant kernel on its own with CUDA events, in the launch shape
    the decode step uses (the same grid: the handle's tiles per split over the step's
    longest row); achieved = algorithmic bytes per launch / mean launch time."""
    import torch
    from transformer_decoder_kv_b200 import attention, attention_workspace_size

    peak, peak_kind = measured_peaks()
    B, H = wl.batch, cfg.n_heads
    # a step of 16 rows or more runs as chains over parts of the rows, each launching the
    # attention over its own rows: time the first chain's launch (the library's split rule)
    split = B >= SPLIT_MIN_BATCH
    n_chains = 1
    if split:
        n_chains, first = chain_rows(B)
        B = first
        lens = list(lens)[:B]
    if cfg.is_whisper:
        name, n_keys, ld = "k_attention (cross-attention, 1500 keys)", [cfg.enc_len] * B, cfg.enc_len
    else:
        n_keys = [int(n) + 1 for n in lens]
        ld = int(max(n_keys))
        name = "k_attention (self-attention over the KV cache)"
    g = torch.Generator(device="cuda")
    g.manual_seed(1)
    q = torch.randn((B, H, 64), device="cuda", generator=g)
    # one buffer per rotation so that every timed launch reads K/V from HBM, not L2
    per = 2 * B * H * ld * 64 * 4
    nbuf = max(2, min(8, int(np.ceil(3 * L2_BYTES / per)) + 1))
    nbuf = min(nbuf, max(1, int(20e9 // per)))
    ks = [torch.randn((B, H, ld, 64), device="cuda", generator=g) for _ in range(nbuf)]
    vs = [torch.randn((B, H, ld, 64), device="cuda", generator=g) for _ in range(nbuf)]
    lens_d = torch.tensor(n_keys, dtype=torch.int32, device="cuda")
    out = torch.empty((B, H, 64), device="cuda")
    wsb = attention_workspace_size(B, H, ld)
    ws = torch.zeros(wsb // 4 + 1, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream()
    for i in range(3):
        attention(q, ks[i % nbuf], vs[i % nbuf], lens_d, B, H, ld, out, ws, wsb, s.cuda_stream, tiles_per_split)
    reps = 20
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for i in range(reps):
        attention(q, ks[i % nbuf], vs[i % nbuf], lens_d, B, H, ld, out, ws, wsb, s.cuda_stream, tiles_per_split)
    e1.record(s)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    alg = sum(n * 64 * 4 * 2 for n in n_keys) * H + 2 * B * H * 64 * 4
    achieved = alg / (ms / 1e3) / 1e9
    traffic = recorded_traffic(wl.name, alg)
    max_tiles = (ld + 63) // 64
    grid = [-(-max_tiles // tiles_per_split), H, B]
    if split:
        name += f", one of the step's {n_chains} chains ({B} of {wl.batch} streams)"
    return {"kernel": name, "grid": grid, "tiles_per_split": tiles_per_split, "bound": "hbm",
            "achieved": round(achieved, 1), "peak": peak,
            "peak_kind": f"{peak_kind} hbm_gbs (copy, burst)", "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": traffic, "algorithmic_bytes": alg,
            "launch_us": round(ms * 1e3, 2)}


def recorded_traffic(wl_name: str, algorithmic_bytes: int):
    """DRAM bytes per launch from the committed ncu summary, if the kernel source is
    unchanged since the capture; otherwise null. A record taken on a smaller case of the
    same launch shape holds DRAM bytes per algorithmic byte, scaled here to this launch."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    rec = d.get(wl_name)
    if not rec:
        return None
    src = os.path.join(ROOT, "transformer_decoder_kv_b200", "csrc", "attention.cuh")
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if rec.get("source_sha") != h:
        return None
    if "dram_per_algorithmic_byte" in rec:
        return int(round(rec["dram_per_algorithmic_byte"] * algorithmic_bytes))
    return rec.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- CPU oracle

def oracle_sample(wl: synth.Workload, seed: int, budget_s: float = 15.0, cores: int = 0) -> dict:
    """Time the CPU oracle on a bounded sample of the workload: the first few streams
    (at their own initial lengths), a few steps. Returns tokens/s and the sample. `cores`
    is the BLAS thread count the caller set for this process (the oracle's arithmetic runs
    in numpy's BLAS)."""
    import oracle

    cfg = wl.model
    W = synth.make_weights(cfg, seed)
    lens = synth.cache_lens(wl, seed)
    n_streams = min(wl.batch, 4 if cfg.n_layers <= 6 else 2)
    ref = oracle.OracleDecoder(W, wl.max_cache_len)
    states = []
    for s in range(n_streams):
        n = int(lens[s])
        enc = synth.encoder_hidden(cfg, s, seed) if cfg.is_whisper else None
        st = ref.new_state(enc)
        if wl.cache_init == "prefill":
            ref.prefill(st, list(synth.token_ids(cfg, s, n, seed)))
        else:
            ks, vs = zip(*(synth.seed_kv(cfg, s, l, n, seed) for l in range(cfg.n_layers)))
            ref.kv_append(st, 0, np.stack(ks), np.stack(vs))
        states.append(st)
    toks = [int(t) for t in synth.token_ids(cfg, 7777, n_streams, seed)]
    t0 = time.perf_counter()
    steps = 0
    while True:
        _, lg = ref.step(states, toks, [st.n for st in states])
        toks = [int(np.argmax(r)) for r in lg]
        steps += 1
        if time.perf_counter() - t0 > budget_s or steps >= wl.steps or any(
                st.n + 1 > wl.max_cache_len for st in states):
            break
    el = time.perf_counter() - t0
    return {"value": n_streams * steps / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{n_streams} of {wl.batch} streams at their seeded cache lengths, {steps} "
                      f"decode steps, numpy f64 oracle ({el:.1f} s)"}


BLAS_ENV = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS", "BLIS_NUM_THREADS")


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_leg(config_key: str, budget_s: float, threads: int, extra: list = ()) -> dict:
    """Run oracle_sample in a child process whose BLAS pools are set to `threads`."""
    env = dict(os.environ)
    for k in BLAS_ENV:
        env[k] = str(threads)
    cmd = [sys.executable, os.path.abspath(__file__), "--oracle-leg", "--config", config_key,
           "--oracle-budget", str(budget_s), "--oracle-threads", str(threads), *extra]
    r = subprocess.run(cmd, env=env, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"oracle leg failed: {r.stderr[-2000:]}")
    return json.loads(r.stdout.strip().splitlines()[-1])


def cpu_baseline(config_key: str, budget_s: float, extra: list = ()) -> dict:
    """The oracle on all host cores, and a single-thread run of the same sample beside it."""
    cores = host_cores()
    allc = oracle_leg(config_key, budget_s, cores, extra)
    one = oracle_leg(config_key, max(3.0, budget_s / 3), 1, extra)
    allc["single_thread_value"] = one["value"]
    allc["single_thread_sample"] = one["sample"]
    return allc


# ---------------------------------------------------------------- distributed plumbing

_PG = None


def _init_dist(world: int):
    global _PG
    if world > 1 and _PG is None:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
        _PG = dist


def _barrier(world):
    if world > 1:
        _PG.barrier()


def _max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64)
    _PG.all_reduce(t, op=_PG.ReduceOp.MAX)
    return float(t.item())


def combine_ranks(ms: float, tokens: int, world: int):
    """Whole-job throughput: every rank's tokens over the slowest rank's device time.
    Returns (tokens/s, max ms, total tokens); every rank takes the same collective steps."""
    ms_max = _max_over_ranks(ms, world)
    tokens_all = _sum_over_ranks(tokens, world)
    return tokens_all / (ms_max / 1e3), ms_max, tokens_all


def _sum_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64)
    _PG.all_reduce(t, op=_PG.ReduceOp.SUM)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=32)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="c4", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-range", action="store_true",
                    help="bracket the timed steps with cudaProfilerStart/Stop (for ncu --profile-from-start off)")
    ap.add_argument("--fast-setup", action="store_true",
                    help="seed caches with N(0,1) K/V instead of prefilling tokens (profiling runs)")
    ap.add_argument("--head", default="exact", choices=["exact", "int8"],
                    help="LM head: exact three-digit split, or int8 with exact re-scoring of the candidates")
    ap.add_argument("--batch", type=int, default=0,
                    help="profiling only: fewer streams than the workload (same model and kernels)")
    ap.add_argument("--max-cache-len", type=int, default=0,
                    help="profiling only: shorter caches, for ncu captures with a small device footprint")
    ap.add_argument("--oracle-leg", action="store_true", help=argparse.SUPPRESS)
    ap.add_argument("--oracle-budget", type=float, default=15.0, help=argparse.SUPPRESS)
    ap.add_argument("--oracle-threads", type=int, default=0, help=argparse.SUPPRESS)
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    wl = synth.workload(CONFIGS[args.config])
    if args.batch or args.max_cache_len:
        # a reduced variant of the workload for profiling captures; named as such
        L = min(args.max_cache_len or wl.max_cache_len, wl.max_cache_len)
        hi = max(1, min(wl.lens_hi, L - wl.steps - 1))
        wl = synth.scaled(wl, name=f"{wl.name} (profiling variant)", batch=args.batch or wl.batch,
                          max_cache_len=L, lens_lo=min(wl.lens_lo, hi), lens_hi=hi,
                          retire_at=min(wl.retire_at, L) if wl.retire_at else wl.retire_at)
    cfg = wl.model
    if args.oracle_leg:
        print(json.dumps(oracle_sample(wl, 0, budget_s=args.oracle_budget, cores=args.oracle_threads)))
        return
    extra = (["--batch", str(args.batch)] if args.batch else []) + \
        (["--max-cache-len", str(args.max_cache_len)] if args.max_cache_len else [])
    config = {"workload": wl.name, "batch": wl.batch, "n_layers": cfg.n_layers, "d_model": cfg.d_model,
              "vocab": cfg.vocab, "proj": cfg.proj_fmt, "cache_init": wl.cache_init,
              "cache_lens": f"U[{wl.lens_lo},{wl.lens_hi}]", "l2": "inputs larger than L2 per step"
              if step_bytes(cfg, synth.cache_lens(wl))["total"] > L2_BYTES else "n/a",
              "parallelism": f"replicas x{args.gpus}",
              "cache_setup": "seeded K/V rows (profiling)" if args.fast_setup else wl.cache_init,
              "fast_setup": bool(args.fast_setup),
              "head": "exact three-digit" if args.head == "exact" else "int8 + exact re-score of candidates"}
    metric = "decode tokens/s (device-timed)"
    if args.impl == "reference":
        if rank != 0:
            return
        cb = cpu_baseline(args.config, max(5.0, min(60.0, float(max(1, args.steps)))), extra)
        # one step = one token for each of the workload's streams, at the oracle's rate
        line = {"impl": "reference", "metric": metric, "value": cb["value"], "unit": "tokens/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(1e3 * wl.batch / cb["value"], 3),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config, "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return
    _init_dist(world)
    r = run_ours(args, wl, rank, world)
    if rank != 0:
        return
    cb = None if args.no_cpu_baseline or world > 1 else cpu_baseline(args.config, 15.0, extra)
    dtype = {"f32": "f32", "w8a8": "int8 weights+activations, int32 acc, f32 elsewhere",
             "w8a32": "int8 weights, f32 activations"}[cfg.proj_fmt]
    peak, kind = measured_peaks()
    line = {"metric": metric, "value": round(r["value"], 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(r["ms"] / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype,
            "data": "synthetic (seeded; random-init weights)", "config": config,
            "step_hbm": {"algorithmic_bytes_per_step": int(r["step_bytes"]),
                         "achieved_GBps": round(r["achieved_gbs"], 1), "peak_GBps": peak,
                         "frac": round(r["achieved_gbs"] / peak, 4), "peak_kind": kind},
            "roofline": r["roofline"], "cpu_baseline": cb, "e2e": r["e2e"], "clocks": r["clocks"],
            "gpu_launches": r["launches"]}
    print(json.dumps(line))


if __name__ == "__main__":
    main()
