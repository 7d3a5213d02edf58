"""The allocation-free attention entry point gives the same result as the regular one.

dec_attention_noalloc is for callers that cannot allocate device memory (a host
framework that owns the whole device, or a latency-critical path that must not
call cudaMalloc); it keeps its split-K scratch in a fixed array inside the
library. This file is collected last so that, run after the other tests, it also
sees the library already loaded and used; it must pass alone as well.
"""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu


def test_noalloc_attention_matches_workspace_entry_point_and_oracle_twice():
    import torch
    from transformer_decoder_kv_b200 import attention, attention_noalloc, attention_workspace_size

    B, H, ld = 5, 4, 700
    lens = torch.tensor([1, 64, 65, 700, 333], dtype=torch.int32, device="cuda")
    ws_bytes = attention_workspace_size(B, H, ld)
    ws = torch.zeros(ws_bytes // 4 + 1, dtype=torch.int32, device="cuda")
    g = torch.Generator(device="cuda")
    for call in range(2):  # two calls in a row: the shared scratch keeps the last call's contents
        g.manual_seed(100 + call)
        q = torch.randn((B, H, 64), device="cuda", generator=g)
        k = torch.randn((B, H, ld, 64), device="cuda", generator=g)
        v = torch.randn((B, H, ld, 64), device="cuda", generator=g)
        ref = torch.empty((B, H, 64), device="cuda")
        got = torch.full((B, H, 64), float("nan"), device="cuda")
        attention(q, k, v, lens, B, H, ld, ref, ws, ws_bytes)
        attention_noalloc(q, k, v, lens, B, H, ld, got)
        torch.cuda.synchronize()
        # the same launch as dec_attention with tiles_per_split = 0: the same bits
        assert np.array_equal(got.cpu().numpy().view(np.uint32), ref.cpu().numpy().view(np.uint32))
        # and the oracle's attention within the kernel-level tolerance
        qn, kn, vn, ln = q.cpu().numpy(), k.cpu().numpy(), v.cpu().numpy(), lens.cpu().numpy()
        for b in range(B):
            n = int(ln[b])
            want = oracle.attention_decode(qn[b], kn[b, :, :n].transpose(1, 0, 2), vn[b, :, :n].transpose(1, 0, 2))
            np.testing.assert_allclose(got.cpu().numpy()[b], want, rtol=1e-5, atol=1e-5)


def test_noalloc_attention_rejects_sizes_beyond_its_scratch():
    import torch
    from transformer_decoder_kv_b200 import DecError, attention_noalloc, binding

    B, H, ld = 65, 16, 8   # batch * heads = 1040 > 1024
    q = torch.zeros((B, H, 64), device="cuda")
    k = torch.zeros((B, H, ld, 64), device="cuda")
    lens = torch.ones(B, dtype=torch.int32, device="cuda")
    out = torch.zeros((B, H, 64), device="cuda")
    with pytest.raises(DecError) as e:
        attention_noalloc(q, k, k, lens, B, H, ld, out)
    assert e.value.status == binding.DEC_EINVAL
    assert "1024" in str(e.value)
