"""The allocation-free decode-attention entry point (needs a B200).

kivi_decode_attention_static_scratch serves callers that cannot allocate
device memory - for example an engine that loads this library as a plugin and
owns all device memory through its own pool allocator.  It keeps its split
partials, tickets and status word in a static device array instead of a
workspace buffer.  Its results are checked against the CPU oracle element by
element (abs 2e-3 + rel 2e-3), on two calls in a row, on a shape whose pairs
are split across many CTAs and just after a residual flush.  This file is named
to be collected last, so a run that stops at the first failure has run every
other test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import synth
from gpu_util import assert_attention_close, load_kivi

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kivi():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return load_kivi()


def _static_call(K, cache, layer, q, sm_scale=0.0):
    S, _ = cache.length(layer)
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device=q.device)
    return K.kivi_decode_attention_static_scratch(
        cache.cfg, cache.records.data_ptr(), cache.resid_k.data_ptr(),
        cache.resid_v.data_ptr(), layer, S, q, out, sm_scale)


@pytest.mark.parametrize("B,Hkv,Hq,bits", [(4, 8, 32, 2), (8, 8, 64, 2), (2, 4, 4, 4)])
def test_static_scratch_matches_the_oracle(kivi, B, Hkv, Hq, bits):
    """Two layers, two calls each in a row (the array keeps the previous call's
    contents), the second one just after a residual flush."""
    gen = torch.Generator().manual_seed(11 + B + Hq)
    D, S0 = 128, 1055  # NG(1055) = 28 with 159 ring tokens: the next append flushes
    cache = kivi.KiviCache(batch=B, num_layers=2, num_kv_heads=Hkv, num_q_heads=Hq,
                           head_dim=D, bits=bits, max_tokens=S0 + 4)
    refs = []
    for layer in range(2):
        sk = torch.exp(torch.randn(Hkv, D, generator=gen))[None, :, None, :]
        k = (torch.randn(B, Hkv, S0, D, generator=gen) * sk).to(torch.bfloat16)
        v = torch.randn(B, Hkv, S0, D, generator=gen).to(torch.bfloat16)
        cache.prefill(layer, k.cuda(), v.cuda())
        ref = O.OracleCache(B, Hkv, D, bits, S0 + 4)
        ref.prefill(synth.bf16_bits(k), synth.bf16_bits(v))
        refs.append(ref)
    for rnd in range(2):
        if rnd == 1:  # append one token to every layer: each flushes a group
            for layer in range(2):
                kn = torch.randn(B, Hkv, D, generator=gen).to(torch.bfloat16)
                vn = torch.randn(B, Hkv, D, generator=gen).to(torch.bfloat16)
                cache.append(layer, kn.cuda(), vn.cuda())
                refs[layer].append(synth.bf16_bits(kn), synth.bf16_bits(vn))
                assert refs[layer].NG == 29
        for layer in range(2):
            q = torch.randn(B, Hq, D, generator=gen).to(torch.bfloat16)
            got = _static_call(kivi, cache, layer, q.cuda()).cpu().numpy()
            expect = refs[layer].attention(synth.bf16_bits(q))
            assert_attention_close(got, expect, f"static scratch B={B} Hq={Hq} layer {layer}")
    assert kivi.kivi_static_scratch_status() == 0
    cache.close()


def test_static_scratch_agrees_with_the_workspace_entry_point(kivi):
    gen = torch.Generator().manual_seed(5)
    B, Hkv, Hq, D = 3, 2, 8, 64
    cache = kivi.KiviCache(batch=B, num_layers=1, num_kv_heads=Hkv, num_q_heads=Hq, head_dim=D,
                           bits=2, max_tokens=700)
    k = torch.randn(B, Hkv, 700, D, generator=gen).to(torch.bfloat16).cuda()
    cache.prefill(0, k, k)
    for _ in range(2):
        q = torch.randn(B, Hq, D, generator=gen).to(torch.bfloat16).cuda()
        a = cache.attend(0, q).cpu().numpy().astype(np.float64)
        b = _static_call(kivi, cache, 0, q).cpu().numpy()
        assert_attention_close(b, a, "static scratch vs workspace")
    assert kivi.kivi_static_scratch_status() == 0
    assert cache.check_device_status() == 0
    cache.close()


def test_static_scratch_rejects_oversized_calls(kivi):
    """Calls whose tickets, or whose grid's partials, do not fit the array are refused
    before any launch."""
    from decode_attention_kivi_b200 import _native as N

    fake = 1 << 20
    # one ticket per (sequence, kv head): 2^21 pairs need 8 MiB of tickets alone
    cfg = kivi.make_config(batch=1 << 15, num_layers=1, num_kv_heads=64, num_q_heads=64,
                           head_dim=128, bits=2, max_tokens=4096)
    rc = N.lib().kivi_decode_attention_static_scratch(ctypes.byref(cfg), fake, fake, fake, 0,
                                                      300, fake, fake, 0.0, None)
    assert N.STATUS[rc] == "KIVI_ERR_SCRATCH_LIMIT"
    # 100,000 pairs of 8 query heads: the grid's partials (8320 bytes per CTA, one
    # CTA per 17 pairs at least) exceed 8 MiB
    cfg = kivi.make_config(batch=12500, num_layers=1, num_kv_heads=8, num_q_heads=64,
                           head_dim=128, bits=2, max_tokens=4096)
    rc = N.lib().kivi_decode_attention_static_scratch(ctypes.byref(cfg), fake, fake, fake, 0,
                                                      300, fake, fake, 0.0, None)
    assert N.STATUS[rc] == "KIVI_ERR_SCRATCH_LIMIT"
    assert kivi.kivi_static_scratch_status() == 0
