"""Whole decode step through the C ABI against the oracle on small models.

Teacher-forced: both sides get the same tokens every step (the oracle's greedy
pick), so one near-tie cannot cascade; greedy picks must agree wherever the
oracle's top-2 margin exceeds the logit tolerance.
"""
import numpy as np
import pytest

import synth
from tests._harness import ATOL, build_pair, check_row, close, step_both

pytestmark = pytest.mark.gpu


def _run(wl_name, steps=None, seed=0):
    """Teacher-forced steps against the oracle (ensemble for W8A8); returns the
    argmax near-tie events."""
    import torch
    wl = synth.workload(wl_name)
    p = build_pair(wl, seed)
    cfg = wl.model
    B = wl.batch
    toks = [int(t) for t in synth.token_ids(cfg, 999, B, seed)]
    events = []
    for t in range(steps or wl.steps):
        lg, am, hid, rl, rh, env_h, env_l = step_both(p, toks)
        for b in range(B):
            ev = check_row(hid[b], lg[b], am[b], rh[b], rl[b], env_h[b], env_l[b],
                           f"{wl_name} step {t} stream {b}")
            if ev:
                events.append(ev)
        toks = [int(np.argmax(rl[b])) for b in range(B)]
    # K/V rows written by prefill and steps agree with the oracle's cache rows
    for slot, st in enumerate(p.states):
        for l in range(cfg.n_layers):
            n = st.n
            ko = torch.empty((n, cfg.kv_dim), device="cuda")
            vo = torch.empty((n, cfg.kv_dim), device="cuda")
            p.gpu.kv_read(slot, l, 0, n, ko, vo)
            torch.cuda.synchronize()
            env_k = max([0.0] + [float(np.abs(sts[slot].k[l][:n] - st.k[l][:n]).max()) for _, sts in p.jrefs])
            env_v = max([0.0] + [float(np.abs(sts[slot].v[l][:n] - st.v[l][:n]).max()) for _, sts in p.jrefs])
            close(ko.cpu().numpy(), st.k[l][:n], atol=ATOL + 2 * env_k, what=f"K cache slot {slot} layer {l}")
            close(vo.cpu().numpy(), st.v[l][:n], atol=ATOL + 2 * env_v, what=f"V cache slot {slot} layer {l}")
    p.gpu.close()
    if events:
        print(f"{wl_name}: near-tie events: {events}")
    return events


@pytest.mark.parametrize("wl_name", ["tiny_whisper_b3", "tiny_qwen2_b3", "tiny_whisper_w8a32_b3",
                                     "small_qwen2_kv_b5", "tiny_whisper_b9", "tiny_whisper_w8a32_b9",
                                     "tiny_qwen2_b9", "mid_whisper_b9", "mid_qwen2_b9", "tiny_qwen2_gqa_b3",
                                     "mid_qwen2_gqa_b9"])
def test_step_matches_oracle(wl_name):
    _run(wl_name)


def test_greedy_continuation_uses_previous_pick():
    """tokens=NULL feeds each slot its previous device argmax (no host round trip)."""
    import torch
    wl = synth.workload("tiny_whisper_b3")
    p = build_pair(wl)
    cfg = wl.model
    B = wl.batch
    toks = [3, 5, 7]
    for t in range(4):
        pos = [st.n for st in p.states]
        logits = torch.empty((B, cfg.vocab), device="cuda")
        am = torch.empty(B, dtype=torch.int32, device="cuda")
        p.gpu.step(B, None, toks if t == 0 else None, pos, pos, logits, am)
        p.gpu.sync()
        _, rl = p.ref.step(p.states, toks, pos)
        close(logits.cpu().numpy(), rl, what=f"step {t}")
        toks = [int(x) for x in am.cpu().numpy()]
    p.gpu.close()


def test_batched_step_equals_solo_bitwise():
    """franken_ocr decoder_qwen2.rs: a stream's logits in the batched step are byte-for-byte
    those of the same stream stepped alone."""
    import torch
    for wl_name in ("tiny_whisper_b3", "tiny_qwen2_b3"):
        wl = synth.workload(wl_name)
        cfg = wl.model
        pa = build_pair(wl)
        solo = [build_pair(wl, streams=[s], max_slots=1) for s in range(wl.batch)]
        toks = [11, 22, 33]
        lg = step_both(pa, toks)[0]
        for s in range(wl.batch):
            l1 = step_both(solo[s], [toks[s]])[0]
            assert np.array_equal(lg[s].view(np.uint32), l1[0].view(np.uint32)), (wl_name, s)
            solo[s].gpu.close()
        pa.gpu.close()


def test_host_step_matches_device_step():
    import torch
    wl = synth.workload("tiny_whisper_b3")
    cfg = wl.model
    a = build_pair(wl)
    b = build_pair(wl)
    toks = [1, 2, 3]
    lg, am = step_both(a, toks)[:2]
    pos = [st.n for st in b.states]
    lh = np.empty((wl.batch, cfg.vocab), np.float32)
    ah = np.empty(wl.batch, np.int32)
    b.gpu.step_host(wl.batch, None, toks, pos, pos, lh, ah)
    assert np.array_equal(lh.view(np.uint32), lg.view(np.uint32))
    assert np.array_equal(ah, am)
    a.gpu.close()
    b.gpu.close()


def test_errors_are_rejected_before_any_work():
    import torch
    from transformer_decoder_kv_b200 import DecError, binding
    wl = synth.workload("tiny_whisper_b3")
    cfg = wl.model
    p = build_pair(wl)
    n = [st.n for st in p.states]

    def status(fn):
        with pytest.raises(DecError) as e:
            fn()
        return e.value.status

    assert status(lambda: p.gpu.step(3, None, [cfg.vocab, 0, 0], n, n)) == binding.DEC_ERANGE
    assert status(lambda: p.gpu.step(3, None, [0, 0, 0], [cfg.max_pos, 0, 0], n)) == binding.DEC_ERANGE
    bad = list(n)
    bad[1] += 1
    assert status(lambda: p.gpu.step(3, None, [0, 0, 0], n, bad)) == binding.DEC_ESTATE
    assert status(lambda: p.gpu.step(2, [1, 1], [0, 0], [n[1]] * 2, [n[1]] * 2)) == binding.DEC_EINVAL
    assert status(lambda: p.gpu.step(0, None, [], [], [])) == binding.DEC_EINVAL
    # the rejected calls changed nothing
    assert [p.gpu.slot_len(s) for s in range(3)] == n
    # a slot that was never prefilled has no cross-attention K/V
    fresh = build_pair(synth.scaled(wl, batch=1), max_slots=2)
    assert status(lambda: fresh.gpu.step(1, [1], [0], [0], [0])) == binding.DEC_ESTATE
    # cache overflow: fill a slot to max_cache_len
    wl2 = synth.scaled(synth.workload("tiny_qwen2_b3"), batch=1, max_cache_len=8, lens_lo=8, lens_hi=8)
    q = build_pair(wl2)
    assert status(lambda: q.gpu.step(1, None, [0], [8], [8])) == binding.DEC_EOVERFLOW
    for x in (p, fresh, q):
        x.gpu.close()


def test_tensor_core_path_is_batch_invariant_bitwise():
    """Batch 9 (two 8-column tiles) and batch 8 (one tile) give the same bits for the
    same stream: each output column of the tensor-core projections depends only on its
    own activation row."""
    for wl_name in ("mid_whisper_b9", "tiny_whisper_w8a32_b9"):
        wl = synth.workload(wl_name)
        p9 = build_pair(wl)
        p8 = build_pair(wl, streams=list(range(8)), max_slots=8)
        toks = list(range(100, 109))
        l9 = step_both(p9, toks)[0]
        l8 = step_both(p8, toks[:8])[0]
        assert np.array_equal(l9[:8].view(np.uint32), l8.view(np.uint32)), wl_name
        p9.gpu.close()
        p8.gpu.close()


def test_w8a8_tensor_core_path_equals_dp4a_path_bitwise():
    """W8A8 products are exact integer sums on both paths (int8 tensor cores from batch 8
    on, dp4a below) and the quantiser is shared, so a stream's hidden state after the
    layers is bit-identical in a batch of 9 and stepped alone."""
    wl = synth.workload("mid_qwen2_b9")
    p9 = build_pair(wl)
    toks = list(range(200, 209))
    h9 = step_both(p9, toks)[2]
    for s in (0, 5, 8):
        p1 = build_pair(wl, streams=[s], max_slots=1)
        h1 = step_both(p1, [toks[s]])[2]
        assert np.array_equal(h9[s].view(np.uint32), h1[0].view(np.uint32)), s
        p1.gpu.close()
    p9.gpu.close()


def test_step_kernel_count_is_reported():
    """dec_step_kernels gives the kernel count of the step's captured graph: positive, the
    same for repeated steps of one shape, and the layer count sets it for a fixed path."""
    wl = synth.workload("tiny_whisper_b3")
    p = build_pair(wl)
    counts = []
    for t in range(3):
        step_both(p, [5, 6, 7])
        counts.append(p.gpu.step_kernels())
    p.gpu.close()
    assert counts[0] > 0 and len(set(counts)) == 1, counts
    # embed, then per layer: q|k|v, self-attention, o, cross q, cross-attention, cross o,
    # fc1, fc2; then the head (which splits the hidden rows itself at batches up to 16)
    assert counts[0] == 1 + wl.model.n_layers * 8 + 1, counts


def test_head_digit_planes_made_in_kernel_or_by_row_kernel_give_same_bits():
    """Up to batch 16 the tensor-core head splits the hidden rows itself; above 16 a row
    kernel does it first. Both call one device function, and the products are exact integer
    sums, so a stream's logits are the same bits in a batch of 17 and in a batch of 9."""
    wl = synth.scaled(synth.workload("mid_whisper_b9"), batch=17)
    p17 = build_pair(wl)
    p9 = build_pair(wl, streams=list(range(9)), max_slots=9)
    toks = list(range(300, 317))
    l17 = step_both(p17, toks)[0]
    l9 = step_both(p9, toks[:9])[0]
    assert np.array_equal(l17[:9].view(np.uint32), l9.view(np.uint32))
    p17.gpu.close()
    p9.gpu.close()


@pytest.mark.parametrize("name,n", [("mid_qwen2", 200), ("small_qwen2", 131), ("mid_whisper", 60),
                                     ("tiny_whisper_w8a32", 50)])
def test_chunked_prefill_equals_row_by_row_prefill(name, n):
    """A prompt run as chunks of rows of one slot (causal attention per row, m = chunk
    projections) fills the same cache and gives the same last logits as one row per step:
    bit for bit for W8A8 (exact integer products, per-row split boundaries), within the
    tolerance for f32 / W8A32 (the split-TF32 path from 8 rows on)."""
    import torch
    from transformer_decoder_kv_b200 import Decoder

    cfg = synth.MODELS[name]
    W = synth.make_weights(cfg, 0)
    n = min(n, cfg.max_pos)
    toks = synth.token_ids(cfg, 3, n)
    enc = torch.from_numpy(synth.encoder_hidden(cfg, 0)).cuda() if cfg.is_whisper else None
    outs = []
    for chunk in (1, 128, 37):
        dec = Decoder(cfg, W, max_slots=2, max_cache_len=256)
        dec.set_prefill_chunk(chunk)
        lg = torch.empty(cfg.vocab, device="cuda")
        dec.prefill(1, toks, enc, lg)
        k = torch.empty((cfg.n_layers, n, cfg.kv_dim), device="cuda")
        v = torch.empty_like(k)
        for l in range(cfg.n_layers):
            dec.kv_read(1, l, 0, n, k[l], v[l])
        nxt = dec.next_tokens([1])[0]
        torch.cuda.synchronize()
        outs.append((lg.cpu().numpy(), k.cpu().numpy(), v.cpu().numpy(), nxt))
        assert dec.slot_len(1) == n
        dec.close()
    base = outs[0]
    for o in outs[1:]:
        if cfg.proj_fmt == "w8a8":
            for a, b in zip(o[:3], base[:3]):
                assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
        else:
            for a, b in zip(o[:3], base[:3]):
                close(a, b, what=name)
        assert o[3] == int(np.argmax(o[0]))


def test_phase_timing_lists_every_phase_and_matches_the_step():
    """dec_phase_times: one entry per phase in launch order (embed, per layer q|k|v,
    self-attention, o, [cross q, cross-attention, cross o,] FFN up, FFN down, then the head),
    positive device times, and the timed step computes the same logits as an untimed one."""
    import torch
    for wl_name in ("tiny_whisper_b3", "tiny_qwen2_b3"):
        wl = synth.workload(wl_name)
        cfg = wl.model
        a, b = build_pair(wl), build_pair(wl)
        b.gpu.set_phase_timing(True)
        toks = [4, 5, 6]
        la = step_both(a, toks)[0]
        lb = step_both(b, toks)[0]
        assert np.array_equal(la.view(np.uint32), lb.view(np.uint32))
        ph = b.gpu.phase_times()
        per_layer = ["qkv", "self_attn", "o"] + (["cross_q", "cross_attn", "cross_o"] if cfg.is_whisper else []) + \
            ["ffn_up", "ffn_down"]
        want = [(-1, "embed")] + [(l, k) for l in range(cfg.n_layers) for k in per_layer] + [(-1, "head")]
        assert [(l, k) for l, k, _ in ph] == want
        assert all(ms > 0 for _, _, ms in ph)
        a.gpu.close()
        b.gpu.close()
