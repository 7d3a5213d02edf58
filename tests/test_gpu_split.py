"""Decode steps of 16 rows or more run as chains (two) over equal parts of the rows, on their
own streams, with no dependency between them (run_step's split). Every output of a row
depends only on that row's own inputs on every path the chains use (exact integer sums for
W8A8, the digit-plane Whisper projections and the head; attention split boundaries fixed per
row), so a split step must give the same bits as the same rows stepped in smaller, unsplit
batches: logits, greedy picks and the K/V rows the step appends, over several steps that feed
their own picks.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


def _prefilled(cfg, W, B, max_len, seed=0):
    import torch
    from transformer_decoder_kv_b200 import Decoder

    dec = Decoder(cfg, W, max_slots=B, max_cache_len=max_len)
    r = np.random.default_rng(seed)
    lens = []
    for s in range(B):
        n = int(r.integers(1, 20))
        enc = torch.from_numpy(synth.encoder_hidden(cfg, s, seed)).cuda() if cfg.is_whisper else None
        dec.prefill(s, [int(t) for t in synth.token_ids(cfg, 300 + s, n, seed)], enc)
        lens.append(n)
    return dec, lens


@pytest.mark.parametrize("name,B", [("mid_qwen2", 40), ("mid_qwen2", 64), ("mid_qwen2_gqa", 33),
                                    ("tiny_whisper_w8a32", 48), ("tiny_whisper", 32)])
def test_split_step_equals_unsplit_groups(name, B):
    import torch

    cfg = synth.MODELS[name]
    W = synth.make_weights(cfg, 0)
    split, lens = _prefilled(cfg, W, B, 64)
    ref, lens2 = _prefilled(cfg, W, B, 64)
    assert lens == lens2
    # unsplit groups of at most 16 rows (Whisper groups of 8 or more stay on the digit path)
    groups = [list(range(i, min(i + 16, B))) for i in range(0, B, 16)]
    assert all(len(gr) < 32 for gr in groups)
    assert not cfg.is_whisper or all(len(gr) >= 8 for gr in groups)
    toks = [int(t) for t in synth.token_ids(cfg, 99, B, 0)]
    for t in range(3):
        pos = list(lens)
        lg = torch.empty((B, cfg.vocab), device="cuda")
        am = torch.empty(B, dtype=torch.int32, device="cuda")
        split.step(B, None, toks, pos, pos, lg, am)
        split.sync()
        lg_ref = torch.empty((B, cfg.vocab), device="cuda")
        am_ref = torch.empty(B, dtype=torch.int32, device="cuda")
        for gr in groups:
            n = len(gr)
            lo = torch.empty((n, cfg.vocab), device="cuda")
            ao = torch.empty(n, dtype=torch.int32, device="cuda")
            ref.step(n, gr, [toks[s] for s in gr], [pos[s] for s in gr], [pos[s] for s in gr], lo, ao)
            ref.sync()
            lg_ref[gr] = lo
            am_ref[gr] = ao
        a, b = lg.cpu().numpy(), lg_ref.cpu().numpy()
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), (name, B, t)
        assert np.array_equal(am.cpu().numpy(), am_ref.cpu().numpy()), (name, B, t)
        toks = [int(x) for x in am.cpu().numpy()]
        lens = [x + 1 for x in lens]
    # the appended K/V rows are the same bits too
    for s in (0, B // 2, B - 1):
        n = lens[s]
        kv = []
        for d in (split, ref):
            k = torch.empty((n, cfg.kv_dim), device="cuda")
            v = torch.empty_like(k)
            d.kv_read(s, cfg.n_layers - 1, 0, n, k, v)
            torch.cuda.synchronize()
            kv.append((k.cpu().numpy(), v.cpu().numpy()))
        assert np.array_equal(kv[0][0].view(np.uint32), kv[1][0].view(np.uint32))
        assert np.array_equal(kv[0][1].view(np.uint32), kv[1][1].view(np.uint32))
    split.close()
    ref.close()
