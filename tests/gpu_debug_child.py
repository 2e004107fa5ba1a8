"""Run by test_gpu_debug.py in a child process whose KIVI_LIBRARY points at the
debug build (libkivi_debug.so): short bounded waits, copy bounds checks, and a
hook that makes the decode kernel's waits run out (not a test module)."""
import sys

import numpy as np
import torch

import oracle as O
import synth
from gpu_util import assert_attention_close, load_kivi


def parity_under_bounds_checks(K):
    """Small edge cases: the bounds-checked build must report nothing and agree
    with the oracle."""
    for S0, steps, D, bits, hpk in [(0, 3, 64, 2, 2), (127, 3, 64, 2, 2), (159, 3, 128, 2, 4),
                                    (255, 40, 64, 2, 2), (700, 2, 128, 4, 4), (512, 1, 64, 2, 8)]:
        gen = torch.Generator().manual_seed(S0 + D + bits)
        B, Hkv = 2, 2
        k = torch.randn(B, Hkv, S0, D, generator=gen).to(torch.bfloat16)
        v = torch.randn(B, Hkv, S0, D, generator=gen).to(torch.bfloat16)
        cache = K.KiviCache(batch=B, num_layers=1, num_kv_heads=Hkv, num_q_heads=Hkv * hpk,
                            head_dim=D, bits=bits, max_tokens=S0 + steps)
        ref = O.OracleCache(B, Hkv, D, bits, S0 + steps)
        if S0:
            cache.prefill(0, k.cuda(), v.cuda())
            ref.prefill(synth.bf16_bits(k), synth.bf16_bits(v))
        for _ in range(steps):
            kn = torch.randn(B, Hkv, D, generator=gen).to(torch.bfloat16)
            vn = torch.randn(B, Hkv, D, generator=gen).to(torch.bfloat16)
            q = torch.randn(B, Hkv * hpk, D, generator=gen).to(torch.bfloat16)
            cache.append(0, kn.cuda(), vn.cuda())
            ref.append(synth.bf16_bits(kn), synth.bf16_bits(vn))
            out = cache.attend(0, q.cuda()).cpu().numpy()
            assert_attention_close(out, ref.attention(synth.bf16_bits(q)), f"bounds build S={ref.S}")
        assert cache.check_device_status() == 0, f"bounds build reported a failure at S0={S0}"
        cache.close()
    print("bounds: ok")


def wait_runs_out(K):
    """Overstated copy sizes: every wait runs out after about 1 ms, the call
    reports KIVI_ERR_DEVICE, and the next normal call is correct."""
    from decode_attention_kivi_b200 import _native as N

    gen = torch.Generator().manual_seed(9)
    B, Hkv, Hq, D = 2, 2, 4, 64
    k = torch.randn(B, Hkv, 700, D, generator=gen).to(torch.bfloat16)
    v = torch.randn(B, Hkv, 700, D, generator=gen).to(torch.bfloat16)
    q = torch.randn(B, Hq, D, generator=gen).to(torch.bfloat16)
    cache = K.KiviCache(batch=B, num_layers=1, num_kv_heads=Hkv, num_q_heads=Hq, head_dim=D,
                        bits=2, max_tokens=700)
    ref = O.OracleCache(B, Hkv, D, 2, 700)
    cache.prefill(0, k.cuda(), v.cuda())
    ref.prefill(synth.bf16_bits(k), synth.bf16_bits(v))
    expect = ref.attention(synth.bf16_bits(q))
    assert_attention_close(cache.attend(0, q.cuda()).cpu().numpy(), expect, "before")
    assert cache.check_device_status() == 0
    assert N.lib().kivi_debug_overstate_copies(16) == 0
    cache.attend(0, q.cuda())
    code = cache.check_device_status()
    assert code & 1, f"the waits did not report running out (status word {code})"
    assert N.lib().kivi_debug_overstate_copies(0) == 0
    assert_attention_close(cache.attend(0, q.cuda()).cpu().numpy(), expect, "after")
    assert cache.check_device_status() == 0
    cache.close()
    print("wait: ok")


if __name__ == "__main__":
    K = load_kivi()
    for name in sys.argv[1:]:
        {"bounds": parity_under_bounds_checks, "wait": wait_runs_out}[name](K)
