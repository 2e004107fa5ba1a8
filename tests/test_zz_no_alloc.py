"""The allocation-free decode-attention entry point (needs a B200).

kivi_decode_attention_static_scratch serves callers that cannot allocate
device memory - for example an engine that loads this library as a plugin and
owns all device memory through its own pool allocator.  It keeps its split-K
partials in a static device array instead of a workspace buffer.  This file is
named to be collected last, so a run that stops at the first failure has run
every other test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ATOL = 2e-3
RTOL = 2e-3


@pytest.fixture(scope="module")
def kivi():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from decode_attention_kivi_b200 import build

    build.build()
    import decode_attention_kivi_b200 as K

    return K


def _static_call(K, cache, layer, q, sm_scale=0.0):
    S, _ = cache.length(layer)
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device=q.device)
    return K.kivi_decode_attention_static_scratch(
        cache.cfg, cache.records.data_ptr(), cache.resid_k.data_ptr(),
        cache.resid_v.data_ptr(), layer, S, q, out, sm_scale)


def test_static_scratch_matches_workspace_entry_point(kivi):
    """Two calls in a row through the C ABI agree with kivi_decode_attention."""
    gen = torch.Generator().manual_seed(11)
    B, Hkv, Hq, D, S0 = 4, 8, 32, 128, 1000
    cache = kivi.KiviCache(batch=B, num_layers=2, num_kv_heads=Hkv, num_q_heads=Hq,
                           head_dim=D, bits=2, max_tokens=S0 + 4)
    for layer in range(2):
        k = torch.randn(B, Hkv, S0, D, generator=gen).to(torch.bfloat16).cuda()
        v = torch.randn(B, Hkv, S0, D, generator=gen).to(torch.bfloat16).cuda()
        cache.prefill(layer, k, v)
    calls = [(0, 0.0), (1, 0.0)]
    for layer, scale in calls:
        q = torch.randn(B, Hq, D, generator=gen).to(torch.bfloat16).cuda()
        ref = cache.attend(layer, q, sm_scale=scale).cpu().numpy().astype(np.float64)
        got = _static_call(kivi, cache, layer, q, scale).cpu().numpy()
        assert np.isfinite(got).all()
        err = np.abs(got - ref)
        assert (err <= ATOL + RTOL * np.abs(ref)).all(), f"layer {layer}: max err {err.max():.3e}"
    # a second pass over the same layer after an append (the array keeps old contents)
    kn = torch.randn(B, Hkv, D, generator=gen).to(torch.bfloat16).cuda()
    cache.append(1, kn, kn)
    q = torch.randn(B, Hq, D, generator=gen).to(torch.bfloat16).cuda()
    ref = cache.attend(1, q).cpu().numpy().astype(np.float64)
    got = _static_call(kivi, cache, 1, q).cpu().numpy()
    assert (np.abs(got - ref) <= ATOL + RTOL * np.abs(ref)).all()
    cache.close()


def test_static_scratch_rejects_oversized_calls(kivi):
    """A call whose fewest splits (one over the groups, five residual chunks) do not fit
    the array is refused before any launch."""
    from decode_attention_kivi_b200 import _native as N

    cfg = kivi.make_config(batch=512, num_layers=1, num_kv_heads=64, num_q_heads=64,
                           head_dim=128, bits=2, max_tokens=4096)
    assert 256 + 6 * 512 * 64 * 130 * 4 > N.STATIC_SCRATCH_BYTES
    fake = 1 << 20
    rc = N.lib().kivi_decode_attention_static_scratch(ctypes.byref(cfg), fake, fake, fake, 0,
                                                      300, fake, fake, 0.0, None)
    assert N.STATUS[rc] == "KIVI_ERR_SCRATCH_LIMIT"
