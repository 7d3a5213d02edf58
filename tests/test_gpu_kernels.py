"""Kernel-level parity through the C ABI: KV append/read bit-exact, int8 dot products
bit-exact, split-K attention against the oracle."""
import numpy as np
import pytest

import oracle
import synth
from tests._harness import close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    assert torch.cuda.is_available()
    return torch


def test_kv_append_then_read_is_bit_exact(torch_cuda):
    torch = torch_cuda
    from transformer_decoder_kv_b200 import Decoder
    cfg = synth.MODELS["small_qwen2"]
    W = synth.make_weights(cfg, 0)
    dec = Decoder(cfg, W, max_slots=3, max_cache_len=300)
    rng = np.random.default_rng(5)
    n0, n1 = 131, 67
    k0 = rng.standard_normal((cfg.n_layers, n0, cfg.d_model)).astype(np.float32)
    v0 = rng.standard_normal((cfg.n_layers, n0, cfg.d_model)).astype(np.float32)
    # special values must survive the copy unchanged
    k0[0, 0, :4] = [np.inf, -np.inf, -0.0, np.float32(1e-45)]
    dec.kv_append(1, 0, n0, torch.from_numpy(k0).cuda(), torch.from_numpy(v0).cuda())
    k1 = rng.standard_normal((cfg.n_layers, n1, cfg.d_model)).astype(np.float32)
    v1 = rng.standard_normal((cfg.n_layers, n1, cfg.d_model)).astype(np.float32)
    dec.kv_append(1, 100, n1, torch.from_numpy(k1).cuda(), torch.from_numpy(v1).cuda())
    assert dec.slot_len(1) == 167
    kexp = np.concatenate([k0[:, :100], k1], axis=1)
    vexp = np.concatenate([v0[:, :100], v1], axis=1)
    for l in range(cfg.n_layers):
        ko = torch.empty((167, cfg.d_model), device="cuda")
        vo = torch.empty((167, cfg.d_model), device="cuda")
        dec.kv_read(1, l, 0, 167, ko, vo)
        torch.cuda.synchronize()
        assert np.array_equal(ko.cpu().numpy().view(np.uint32), kexp[l].view(np.uint32))
        assert np.array_equal(vo.cpu().numpy().view(np.uint32), vexp[l].view(np.uint32))
    dec.close()


@pytest.mark.parametrize("m,n,k", [(1, 1, 16), (1, 1031, 1024), (3, 77, 2816), (16, 300, 512),
                                   (17, 129, 1280), (64, 96, 2816)])
def test_i8_dot_is_bit_exact(torch_cuda, m, n, k):
    torch = torch_cuda
    from transformer_decoder_kv_b200 import i8_dot
    rng = np.random.default_rng(m * 1000 + n)
    xq = rng.integers(-127, 128, size=(m, k)).astype(np.int8)
    wq = rng.integers(-127, 128, size=(n, k)).astype(np.int8)
    xq[0, :16] = 127
    wq[0, :16] = -127
    acc = torch.empty((m, n), dtype=torch.int32, device="cuda")
    i8_dot(torch.from_numpy(xq).cuda(), torch.from_numpy(wq).cuda(), m, n, k, acc)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), oracle.int8_dot_acc(xq, wq))


@pytest.mark.parametrize("m", [8, 16, 17, 32, 64])
@pytest.mark.parametrize("n,k", [(3072, 1024), (5632, 1024), (1024, 2816), (200, 384)])
def test_i8_dot_tcgen05_is_bit_exact(torch_cuda, m, n, k):
    """The tcgen05 kind::i8 kernel the W8A8 step uses from batch 8 on: its int32
    accumulators (TMEM, split-K partials added by the last arriving warp) equal the
    exact integer dot products, including the largest magnitudes (127 * 127 * K)."""
    torch = torch_cuda
    from transformer_decoder_kv_b200 import i8_dot
    rng = np.random.default_rng(m * 7919 + n + k)
    xq = rng.integers(-127, 128, size=(m, k)).astype(np.int8)
    wq = rng.integers(-127, 128, size=(n, k)).astype(np.int8)
    xq[0, :] = 127
    wq[0, :] = 127
    wq[1, :] = -127
    acc = torch.full((m, n), -1, dtype=torch.int32, device="cuda")
    i8_dot(torch.from_numpy(xq).cuda(), torch.from_numpy(wq).cuda(), m, n, k, acc, path="tcgen05")
    torch.cuda.synchronize()
    want = oracle.int8_dot_acc(xq, wq)
    assert want[0, 0] == 127 * 127 * k
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), want)


@pytest.mark.parametrize("lens,ld", [([1, 0, 64, 65], 80), ([31, 1500, 7], 1500),
                                     ([4129, 128, 2000, 4096], 4129)])
def test_attention_op_matches_oracle(torch_cuda, lens, ld):
    torch = torch_cuda
    from transformer_decoder_kv_b200 import attention, attention_workspace_size
    B, H = len(lens), 3
    rng = np.random.default_rng(sum(lens))
    q = rng.standard_normal((B, H, 64)).astype(np.float32)
    k = rng.standard_normal((B, H, ld, 64)).astype(np.float32)
    v = rng.standard_normal((B, H, ld, 64)).astype(np.float32)
    out = torch.full((B, H, 64), float("nan"), device="cuda")
    ws_bytes = attention_workspace_size(B, H, ld)
    ws = torch.zeros(ws_bytes // 4 + 1, dtype=torch.int32, device="cuda")
    args = (torch.from_numpy(q).cuda(), torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(),
            torch.tensor(lens, dtype=torch.int32, device="cuda"))
    for _ in range(2):  # the second call checks the arrival counters were reset
        attention(*args, B, H, ld, out, ws, ws_bytes)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        for b in range(B):
            n = lens[b]
            if n == 0:
                assert np.array_equal(got[b], np.zeros((H, 64), np.float32))
                continue
            ref = oracle.attention_decode(q[b], k[b, :, :n].transpose(1, 0, 2), v[b, :, :n].transpose(1, 0, 2))
            close(got[b], ref, atol=1e-5, rtol=1e-5, what=f"attention b={b} n={n}")


def test_attention_op_nan_row_fails_closed(torch_cuda):
    torch = torch_cuda
    from transformer_decoder_kv_b200 import attention, attention_workspace_size
    B, H, ld = 2, 1, 300
    rng = np.random.default_rng(1)
    q = rng.standard_normal((B, H, 64)).astype(np.float32)
    k = rng.standard_normal((B, H, ld, 64)).astype(np.float32)
    v = rng.standard_normal((B, H, ld, 64)).astype(np.float32)
    k[0, 0, 123, 5] = np.nan
    out = torch.empty((B, H, 64), device="cuda")
    ws_bytes = attention_workspace_size(B, H, ld)
    ws = torch.zeros(ws_bytes // 4 + 1, dtype=torch.int32, device="cuda")
    attention(torch.from_numpy(q).cuda(), torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(),
              torch.tensor([ld, ld], dtype=torch.int32, device="cuda"), B, H, ld, out, ws, ws_bytes)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    assert np.array_equal(got[0], np.zeros((H, 64), np.float32))
    ref = oracle.attention_decode(q[1], k[1].transpose(1, 0, 2), v[1].transpose(1, 0, 2))
    close(got[1], ref, atol=1e-5, rtol=1e-5)
