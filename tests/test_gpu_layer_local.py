"""Layer-local parity through the C ABI (see tests/_layer_local.py).

Each layer of the CUDA decoder is compared with the oracle's same layer run from the GPU's
own input residual and cache rows, at the plain tolerance (2e-3 abs + 1e-3 rel) except
where an int8 activation on a rounding tie (W8A8 only) reaches the element, in which case
the allowance grows by exactly what rounding that activation the other way changes. The
mutation tests plant a mistake in the oracle (a dropped q bias, RoPE one position off) and
require the same check to fail.
"""
import numpy as np
import pytest

import synth
from tests._layer_local import run_layer_local

pytestmark = pytest.mark.gpu


def _check(rep, whisper):
    print(f"layers {rep.layers} elements {rep.elements} ties {rep.ties} enveloped {rep.enveloped} "
          f"beyond plain tolerance {rep.beyond_tol} max error without a tie {rep.max_err_no_tie:.3g} "
          f"max envelope {rep.max_env:.3g} tight-tolerance misses {len(rep.tight_violations)}")
    print(rep.tight_violations[:5])
    assert not rep.violations, rep.violations[:5]
    if whisper:
        # f32 models have no quantiser: every element meets the plain tolerance
        assert rep.ties == 0 and rep.enveloped == 0 and rep.beyond_tol == 0


@pytest.mark.parametrize("wl_name,steps", [("small_qwen2_kv_b5", 3), ("mid_qwen2_b9", 2), ("tiny_qwen2_b9", 2),
                                           ("tiny_whisper_b3", 2), ("mid_whisper_b9", 2),
                                           ("tiny_whisper_w8a32_b9", 2), ("mid_qwen2_gqa_b9", 2),
                                           ("tiny_qwen2_gqa_b3", 2)])
def test_layer_local_small_models(wl_name, steps):
    wl = synth.workload(wl_name)
    rep = run_layer_local(wl_name, steps, sample=list(range(wl.batch)))
    _check(rep, wl.model.is_whisper)


def test_layer_local_c3_qwen2_b1():
    _check(run_layer_local("c3_qwen2_0_5b_int8_b1", 2, sample=[0]), False)


def test_layer_local_c4_qwen2_b64():
    wl = synth.workload("c4_qwen2_0_5b_int8_b64")
    lens = synth.cache_lens(wl, 0)
    _check(run_layer_local(wl.name, 1, sample=sorted({int(np.argmin(lens)), int(np.argmax(lens))})), False)


def test_layer_local_c1_whisper_tiny_block():
    _check(run_layer_local("c1_whisper_tiny_block_b1", 2, sample=[0]), True)


def test_layer_local_c5_whisper_large_v3_w8a32_b32():
    wl = synth.workload("c5_whisper_large_v3_w8a32_b32")
    lens = synth.cache_lens(wl, 0)
    _check(run_layer_local(wl.name, 1, sample=sorted({int(np.argmin(lens)), int(np.argmax(lens))})), True)


def _drop_q_bias(W):
    for L in W["layers"]:
        L["q"]["b"] = np.zeros_like(L["q"]["b"])
    return W


@pytest.mark.parametrize("wl_name", ["mid_qwen2_b9", "c4_qwen2_0_5b_int8_b64", "mid_whisper_b9"])
def test_layer_local_detects_a_dropped_q_bias(wl_name):
    """The oracle with its q bias removed (a planted mistake) must fail the same check."""
    wl = synth.workload(wl_name)
    sample = [0, 1] if wl.batch > 2 else [0]
    rep = run_layer_local(wl_name, 1, sample=sample, mutate=_drop_q_bias)
    print(rep.violations[:3], rep.tight_violations[:3])
    assert rep.violations or rep.tight_violations


@pytest.mark.parametrize("wl_name", ["mid_qwen2_b9", "c4_qwen2_0_5b_int8_b64"])
def test_layer_local_detects_rope_one_position_off(wl_name):
    """The oracle rotating q and k at position + 1 (a planted mistake) must fail the same check."""
    rep = run_layer_local(wl_name, 1, sample=[0, 1], position_shift=1)
    print(rep.violations[:3])
    assert rep.violations
