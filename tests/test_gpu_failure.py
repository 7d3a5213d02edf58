"""Failure detection without a device fault (lattice-inference cpu_q8.rs: fail closed and
report, never hang; cera whisper.rs: errors instead of undefined results).

* A bounded device wait runs out: a host-side injection makes one attention CTA announce a
  K/V tile on its mbarrier without issuing the copy, so the wait can only expire (after a
  1 ms limit). The kernel returns, the step reports DEC_ETIMEOUT, the handle refuses further
  work until dec_reset, and after the reset and a new prefill the decoder matches the oracle
  again (the arrival counters were left consistent).
* An allocation fails inside dec_create (the n-th one, injected on the host): DEC_ENOMEM,
  no handle, and no device memory left behind.
"""
import numpy as np
import pytest

import oracle
import synth
from tests._harness import close

pytestmark = pytest.mark.gpu


def _prefilled(cfg, W, n_slots, n_tok, max_len=64):
    import torch
    from transformer_decoder_kv_b200 import Decoder

    dec = Decoder(cfg, W, max_slots=n_slots, max_cache_len=max_len)
    for s in range(n_slots):
        enc = synth.encoder_hidden(cfg, s) if cfg.is_whisper else None
        dec.prefill(s, synth.token_ids(cfg, s, n_tok), torch.from_numpy(enc).cuda() if enc is not None else None)
    return dec


@pytest.mark.parametrize("name", ["tiny_qwen2", "tiny_whisper"])
def test_bounded_wait_runs_out_reports_and_recovers(name):
    import torch
    from transformer_decoder_kv_b200 import DecError, binding

    cfg = synth.MODELS[name]
    W = synth.make_weights(cfg, 0)
    dec = _prefilled(cfg, W, 2, 5)
    dec.set_wait_limit(1_000_000)   # 1 ms
    dec.debug_inject(binding.DEC_INJECT_DROP_ATTN_COPY, 1)
    logits = torch.empty((2, cfg.vocab), device="cuda")
    dec.step(2, None, [1, 2], [5, 5], [5, 5], logits)
    with pytest.raises(DecError) as e:
        dec.sync()
    assert e.value.status == binding.DEC_ETIMEOUT
    # the handle refuses work until it is reset
    with pytest.raises(DecError) as e:
        dec.step(2, None, [1, 2], [6, 6], [6, 6], logits)
    assert e.value.status == binding.DEC_ETIMEOUT
    with pytest.raises(DecError) as e:
        dec.prefill(0, [1, 2, 3])
    assert e.value.status == binding.DEC_ETIMEOUT
    # dec_step_host notices a give-up by itself
    dec.debug_inject(binding.DEC_INJECT_DROP_ATTN_COPY, 0)
    dec.reset()
    assert dec.slot_len(0) == 0 and dec.slot_len(1) == 0
    dec.debug_inject(binding.DEC_INJECT_DROP_ATTN_COPY, 1)
    enc = [synth.encoder_hidden(cfg, s) if cfg.is_whisper else None for s in range(2)]
    toks = [synth.token_ids(cfg, s, 5) for s in range(2)]
    for s in range(2):
        dec.prefill(s, toks[s][:0], torch.from_numpy(enc[s]).cuda() if enc[s] is not None else None)
        dec.kv_append(s, 0, 0, None, None)
    with pytest.raises(DecError) as e:
        dec.step_host(1, [0], [3], [0], [0], np.empty((1, cfg.vocab), np.float32), np.empty(1, np.int32))
    assert e.value.status == binding.DEC_ETIMEOUT
    dec.debug_inject(binding.DEC_INJECT_DROP_ATTN_COPY, 0)
    dec.reset()
    # after the reset the decoder works and matches the oracle (counters consistent)
    ref = oracle.OracleDecoder(W, 64)
    states = []
    for s in range(2):
        dec.prefill(s, toks[s], torch.from_numpy(enc[s]).cuda() if enc[s] is not None else None)
        st = ref.new_state(enc[s])
        ref.prefill(st, list(toks[s]))
        states.append(st)
    for t in range(3):
        pos = [st.n for st in states]
        dec.step(2, None, [7 + t, 9 + t], pos, pos, logits)
        dec.sync()
        _, rl = ref.step(states, [7 + t, 9 + t], pos)
        close(logits.cpu().numpy(), rl, what=f"{name} step {t} after reset")
    dec.close()


def test_allocation_failure_in_create_frees_everything():
    import torch
    from transformer_decoder_kv_b200 import DecError, Decoder, binding, debug_fail_alloc

    cfg = synth.MODELS["tiny_qwen2"]
    W = synth.make_weights(cfg, 0)
    torch.cuda.synchronize()
    # a first handle warms up the context and every kernel attribute
    Decoder(cfg, W, max_slots=2, max_cache_len=32).close()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for nth in (1, 2, 7, 25, 60):
        debug_fail_alloc(nth)
        try:
            d = Decoder(cfg, W, max_slots=2, max_cache_len=32)
        except DecError as e:
            assert e.status == binding.DEC_ENOMEM, (nth, str(e))
            assert "injected" in str(e)
        else:
            # fewer allocations than nth: the handle was built; nothing was injected
            d.close()
        torch.cuda.synchronize()
        free = torch.cuda.mem_get_info()[0]
        assert abs(free - free0) <= 4 << 20, (nth, free0 - free)
    # the hook covers one dec_create only
    debug_fail_alloc(0)
    Decoder(cfg, W, max_slots=2, max_cache_len=32).close()
