"""The benchmark's algorithmic bytes per decode step (the denominator of every reported HBM
fraction): each weight once, the tied head, self K/V read and rows written, cross K/V, logits
and embeddings -- checked term by term on a hand-computed configuration and against the
whisper-tiny block's 92.9 MB per step (79.7 MB of it the f32 head)."""
import dataclasses

import numpy as np
import pytest

import bench
import synth


def test_hand_computed_whisper_step():
    cfg = dataclasses.replace(synth.MODELS["tiny_whisper"], n_layers=1, d_model=64, n_heads=1,
                              d_ff=256, vocab=100, enc_len=10)
    b = bench.step_bytes(cfg, np.array([3]))
    # q,k,v,o, cross q,o (6 d^2) + fc1, fc2 (2 d F), f32
    weights = (4 * 64 * 64 + 2 * 64 * 64 + 2 * 64 * 256) * 4
    weights += (6 * 64 + 256 + 64) * 4        # biases of those projections
    weights += 3 * 2 * 64 * 4                 # three LayerNorms (gain, bias)
    assert b["weights"] == weights
    assert b["head"] == 100 * 64 * 4
    assert b["self_kv"] == (3 + 1) * 64 * 2 * 4
    assert b["cross"] == 10 * 64 * 2 * 4
    kv_write, logits, emb = 64 * 2 * 4, 100 * 4, 2 * 64 * 4
    assert b["total"] == weights + b["head"] + b["self_kv"] + kv_write + b["cross"] + logits + emb


def test_hand_computed_qwen2_w8a8_step_counts_scales_and_qkv_bias():
    cfg = dataclasses.replace(synth.MODELS["tiny_qwen2"], n_layers=1, d_model=64, n_heads=1,
                              d_ff=128, vocab=50)
    b = bench.step_bytes(cfg, np.array([5, 7]))
    nW = 4 * 64 * 64 + 3 * 64 * 128                     # int8 codes
    scales = (4 * 64 + 2 * 128 + 64) * 4                 # one f32 per output row
    norms = 2 * 64 * 4
    qkv_bias = 3 * 64 * 4
    assert b["weights"] == nW + scales + norms + qkv_bias
    assert b["self_kv"] == (6 + 8) * 64 * 2 * 4
    assert b["cross"] == 0


def test_whisper_tiny_block_moves_92_9_mb_per_step():
    wl = synth.workload("c1_whisper_tiny_block_b1")
    b = bench.step_bytes(wl.model, synth.cache_lens(wl))
    assert b["head"] == 51865 * 384 * 4
    assert b["total"] == pytest.approx(92.9e6, rel=2e-3)
