"""The int8 LM head with exact refine (franken_ocr decoder_qwen2.rs `LmHead` int8 arm and
`got_lm_head`: int8 per-row head, then an exact re-score of the best candidates).

Two decoders on the same weights and inputs, one with the exact three-digit head and one
with DEC_HEAD_INT8_REFINE, step with the same tokens. The int8 head's candidates are every
token whose coarse logit is within the proven bound of the row's best, so its greedy pick
must equal the exact head's at every step and row, and the logits it re-scored must be the
exact head's bits; elsewhere its logits are the coarse ones.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


def _pair(wl, seed=0):
    import torch
    from transformer_decoder_kv_b200 import Decoder

    cfg = wl.model
    W = synth.make_weights(cfg, seed)
    decs = [Decoder(cfg, W, max_slots=wl.batch, max_cache_len=wl.max_cache_len, head=h) for h in ("exact", "int8")]
    lens = synth.cache_lens(wl, seed)
    g = torch.Generator(device="cuda")
    for s in range(wl.batch):
        n = int(lens[s])
        enc = torch.from_numpy(synth.encoder_hidden(cfg, s, seed)).cuda() if cfg.is_whisper else None
        if wl.cache_init == "prefill":
            toks = synth.token_ids(cfg, s, n, seed)
            for d in decs:
                d.prefill(s, toks, enc)
        else:
            g.manual_seed(1000 + s)
            k = torch.randn((cfg.n_layers, n, cfg.kv_dim), device="cuda", generator=g)
            v = torch.randn((cfg.n_layers, n, cfg.kv_dim), device="cuda", generator=g)
            for d in decs:
                if cfg.is_whisper:
                    d.prefill(s, [], enc)
                d.kv_append(s, 0, n, k, v)
    return decs, lens.astype(np.int64)


@pytest.mark.parametrize("wl_name,steps", [("tiny_qwen2_b3", 4), ("tiny_whisper_b9", 3), ("mid_qwen2_b9", 3),
                                           ("c1_whisper_tiny_block_b1", 1), ("c3_qwen2_0_5b_int8_b1", 3),
                                           ("c4_qwen2_0_5b_int8_b64", 2)])
def test_int8_head_picks_equal_exact_head(wl_name, steps):
    import torch

    wl = synth.workload(wl_name)
    cfg = wl.model
    (ex, i8), lens = _pair(wl)
    B = wl.batch
    toks = [int(t) for t in synth.token_ids(cfg, 77, B, 0)]
    n_cand = []
    for t in range(steps):
        pos = [int(x) for x in lens]
        out = []
        for d in (ex, i8):
            lg = torch.empty((B, cfg.vocab), device="cuda")
            am = torch.empty(B, dtype=torch.int32, device="cuda")
            d.step(B, None, toks, pos, pos, lg, am)
            d.sync()
            out.append((lg.cpu().numpy(), am.cpu().numpy()))
        (le, ae), (li, ai) = out
        assert np.array_equal(ae, ai), (wl_name, t)
        for b in range(B):
            same = le[b].view(np.uint32) == li[b].view(np.uint32)
            assert same[int(ae[b])], (wl_name, t, b)     # the pick was re-scored exactly
            n_cand.append(int(same.sum()))
            # elsewhere the coarse logits stay close to the exact ones
            assert np.abs(le[b].astype(np.float64) - li[b]).max() < 0.1 * max(1.0, np.abs(le[b]).max())
        toks = [int(x) for x in ae]
        lens += 1
    print(f"{wl_name}: exactly re-scored tokens per row: median {np.median(n_cand)}, max {max(n_cand)}")
    ex.close()
    i8.close()


def test_int8_head_with_null_logits_and_generation():
    """Without a caller logits buffer the handle keeps the coarse logits itself; greedy
    generation with the int8 head gives the exact head's tokens."""
    from transformer_decoder_kv_b200 import Decoder

    cfg = synth.MODELS["mid_qwen2"]
    W = synth.make_weights(cfg, 0)
    reqs = [{"prompt": [int(t) for t in synth.token_ids(cfg, i, 5 + 3 * i)], "max_new": 12} for i in range(6)]
    outs = []
    for head in ("exact", "int8"):
        d = Decoder(cfg, W, max_slots=4, max_cache_len=64, head=head)
        outs.append(d.generate(reqs, max_active=4))
        d.close()
    assert outs[0] == outs[1]
