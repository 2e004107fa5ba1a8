"""Helpers shared by the GPU parity tests (not a test module).

Comparison rules: packed records and the bf16 residual ring match the oracle
byte for byte; attention outputs satisfy |gpu - oracle| <= 2e-3 + 2e-3 |oracle|
elementwise (abs 2e-3 / rel 2e-3).
"""
import numpy as np
import torch

import oracle as O
import synth

ATOL = 2e-3
RTOL = 2e-3


def load_kivi():
    """The CUDA library's binding (built in-tree); raises if it cannot be built."""
    from decode_attention_kivi_b200 import build

    build.build()
    import decode_attention_kivi_b200 as K

    return K


def assert_attention_close(gpu: np.ndarray, ref: np.ndarray, what=""):
    err = np.abs(gpu.astype(np.float64) - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    assert not np.isnan(gpu).any(), f"{what}: NaN in GPU output"
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance, "
                           f"max err {err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}")


def assert_state_equal(cache, layer, ref: O.OracleCache, what=""):
    """Records of the NG quantized groups and the live ring slots, byte for byte."""
    S, NG = cache.length(layer)
    assert (S, NG) == (ref.S, ref.NG), what
    if NG:
        got = cache.records_view(layer)[:, :, :NG].cpu().numpy()
        exp = ref.records[:, :, :NG]
        if not np.array_equal(got, exp):
            diff = np.argwhere(got != exp)
            raise AssertionError(f"{what}: {len(diff)} record bytes differ, first at {diff[0]}")
    for t in range(NG * O.G, S):
        slot = t % (O.R + O.G)
        for which, arr in (("k", ref.ring_k), ("v", ref.ring_v)):
            got = synth.bf16_bits(cache.ring_view(which, layer)[:, :, slot])
            assert np.array_equal(got, arr[:, :, slot]), f"{what}: ring {which} token {t}"


def run_sequence(K, k_pre, v_pre, steps_kv, queries, bits, *, Hq, sm_scale=0.0,
                 check_state=True, what=""):
    """Prefill (k_pre, v_pre: bf16 [B][Hkv][S0][D]), then for each step append
    steps_kv[i] = (k_new, v_new) and attend with queries[i] (bf16 [B][Hq][D]),
    on the GPU and in the oracle side by side.  Records and ring are compared
    after the prefill and after every append; attention after every append."""
    B, Hkv, S0, D = k_pre.shape
    max_tokens = max(S0 + len(steps_kv), 1)
    cache = K.KiviCache(batch=B, num_layers=1, num_kv_heads=Hkv, num_q_heads=Hq, head_dim=D,
                        bits=bits, max_tokens=max_tokens)
    ref = O.OracleCache(B, Hkv, D, bits, max_tokens)
    if S0:
        cache.prefill(0, k_pre.cuda(), v_pre.cuda())
        ref.prefill(synth.bf16_bits(k_pre), synth.bf16_bits(v_pre))
        torch.cuda.synchronize()
        if check_state:
            assert_state_equal(cache, 0, ref, f"{what} after prefill S={S0}")
    outs = []
    for (kn, vn), q in zip(steps_kv, queries):
        cache.append(0, kn.cuda(), vn.cuda())
        ref.append(synth.bf16_bits(kn), synth.bf16_bits(vn))
        out = cache.attend(0, q.cuda(), sm_scale=sm_scale).cpu().numpy()
        expect = ref.attention(synth.bf16_bits(q), sm_scale=sm_scale if sm_scale > 0 else None)
        assert_attention_close(out, expect, f"{what} S={ref.S}")
        if check_state:
            assert_state_equal(cache, 0, ref, f"{what} after append S={ref.S}")
        outs.append((out, expect))
    assert cache.check_device_status() == 0
    cache.close()
    return outs
