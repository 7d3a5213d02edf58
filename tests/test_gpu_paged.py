"""Paged self-attention cache (whisper-apr decoder_generated.rs, `PagedDecoderKVCache` /
`forward_one_paged`): a pool of fixed-size pages shared by all slots through a page table.

The page layout changes where rows live, not what is computed, so a paged handle must give
the same bits as a dense one for the same inputs: cache contents, logits and greedy picks,
across seeding, chunked prefill and decode steps with pages started mid-step. A request that
needs more pages than are free is refused before any work, and released slots return their
pages.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


def _handles(wl, page_rows, kv_pages, seed=0):
    import torch
    from transformer_decoder_kv_b200 import Decoder

    cfg = wl.model
    W = synth.make_weights(cfg, seed)
    dense = Decoder(cfg, W, max_slots=wl.batch, max_cache_len=wl.max_cache_len)
    paged = Decoder(cfg, W, max_slots=wl.batch, max_cache_len=wl.max_cache_len, kv_page_rows=page_rows,
                    kv_pages=kv_pages)
    lens = synth.cache_lens(wl, seed)
    for s in range(wl.batch):
        n = int(lens[s])
        enc = torch.from_numpy(synth.encoder_hidden(cfg, s, seed)).cuda() if cfg.is_whisper else None
        if wl.cache_init == "prefill":
            toks = synth.token_ids(cfg, s, n, seed)
            for d in (dense, paged):
                d.prefill(s, toks, enc)
        else:
            ks, vs = zip(*(synth.seed_kv(cfg, s, l, n, seed) for l in range(cfg.n_layers)))
            k, v = torch.from_numpy(np.stack(ks)).cuda(), torch.from_numpy(np.stack(vs)).cuda()
            for d in (dense, paged):
                if cfg.is_whisper:
                    d.prefill(s, [], enc)
                d.kv_append(s, 0, n, k, v)
    return dense, paged, lens.astype(np.int64)


@pytest.mark.parametrize("wl_name,page_rows", [("small_qwen2_kv_b5", 16), ("small_qwen2_kv_b5", 64),
                                               ("tiny_whisper_b3", 16), ("mid_qwen2_gqa_b9", 32),
                                               ("mid_qwen2_b9", 16)])
def test_paged_cache_gives_the_dense_bits(wl_name, page_rows):
    import torch

    wl = synth.workload(wl_name)
    cfg = wl.model
    pages = wl.batch * ((wl.max_cache_len + page_rows - 1) // page_rows)
    dense, paged, lens = _handles(wl, page_rows, pages)
    B = wl.batch
    toks = [int(t) for t in synth.token_ids(cfg, 55, B, 0)]
    for t in range(3):
        pos = [int(x) for x in lens]
        out = []
        for d in (dense, paged):
            lg = torch.empty((B, cfg.vocab), device="cuda")
            am = torch.empty(B, dtype=torch.int32, device="cuda")
            d.step(B, None, toks, pos, pos, lg, am)
            d.sync()
            out.append((lg.cpu().numpy(), am.cpu().numpy()))
        assert np.array_equal(out[0][0].view(np.uint32), out[1][0].view(np.uint32)), (wl_name, t)
        toks = [int(x) for x in out[0][1]]
        lens += 1
    for s in range(B):
        n = int(lens[s])
        for l in (0, cfg.n_layers - 1):
            kv = []
            for d in (dense, paged):
                k = torch.empty((n, cfg.kv_dim), device="cuda")
                v = torch.empty_like(k)
                d.kv_read(s, l, 0, n, k, v)
                torch.cuda.synchronize()
                kv.append((k.cpu().numpy(), v.cpu().numpy()))
            assert np.array_equal(kv[0][0].view(np.uint32), kv[1][0].view(np.uint32))
            assert np.array_equal(kv[0][1].view(np.uint32), kv[1][1].view(np.uint32))
    dense.close()
    paged.close()


def test_paged_pool_exhaustion_is_refused_and_release_returns_pages():
    import torch
    from transformer_decoder_kv_b200 import DecError, Decoder, binding

    cfg = synth.MODELS["tiny_qwen2"]
    W = synth.make_weights(cfg, 0)
    d = Decoder(cfg, W, max_slots=3, max_cache_len=96, kv_page_rows=16, kv_pages=4)
    assert d.kv_pages_free() == 4
    d.prefill(0, synth.token_ids(cfg, 0, 32))          # 2 pages
    d.prefill(1, synth.token_ids(cfg, 1, 20))          # 2 pages
    assert d.kv_pages_free() == 0
    # slot 0 holds 32 rows: its next row starts a third page, and none is free
    with pytest.raises(DecError) as e:
        d.step(2, [0, 1], [3, 4], [32, 20], [32, 20])
    assert e.value.status == binding.DEC_ENOMEM
    assert d.slot_len(0) == 32 and d.slot_len(1) == 20 and d.kv_pages_free() == 0
    with pytest.raises(DecError) as e:
        d.prefill(2, synth.token_ids(cfg, 2, 5))
    assert e.value.status == binding.DEC_ENOMEM
    d.release_slot(1)
    assert d.kv_pages_free() == 2 and d.slot_len(1) == 0
    d.step(1, [0], [3], [32], [32])
    d.sync()
    assert d.kv_pages_free() == 1 and d.slot_len(0) == 33
    d.close()


def test_generate_with_a_small_paged_pool_matches_dense():
    """14 requests through a pool that holds a few streams at a time: admission waits for
    pages, retirement returns them, and every request's tokens equal the dense handle's."""
    from transformer_decoder_kv_b200 import Decoder

    cfg = synth.MODELS["mid_qwen2"]
    W = synth.make_weights(cfg, 0)
    r = np.random.default_rng(4)
    reqs = [{"prompt": [int(t) for t in synth.token_ids(cfg, 900 + i, int(r.integers(1, 40)))],
             "max_new": int(r.integers(1, 25))} for i in range(14)]
    dense = Decoder(cfg, W, max_slots=8, max_cache_len=64)
    want = dense.generate(reqs, max_active=8)
    dense.close()
    paged = Decoder(cfg, W, max_slots=8, max_cache_len=64, kv_page_rows=16, kv_pages=9)
    got = paged.generate(reqs, max_active=8)
    assert got == want
    assert paged.kv_pages_free() == 9
    paged.close()
