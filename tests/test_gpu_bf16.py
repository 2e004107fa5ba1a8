"""Decode attention over an unquantized bf16 cache (needs a B200): the 16-bit
baseline, checked element by element against the oracle's textbook attention.

Tolerance, from the kernel's arithmetic: the scores are exact bf16 products
summed in fp32; p enters P.V as a bf16 pair hi + lo, within 2^-16 of p relative;
the sum of p and the output stay fp32.  So |out - exact| <= 2^-16 max|v| plus
fp32 rounding, under 1e-4 for the unit-normal values here: the bar is
|gpu - oracle| <= 2e-4 + 2e-4 |oracle|.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from gpu_util import load_kivi

pytestmark = pytest.mark.gpu
TOL = 2e-4


@pytest.fixture(scope="module")
def kivi():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return load_kivi()


def _close(got, ref, what):
    err = np.abs(got.astype(np.float64) - ref)
    bad = err > TOL + TOL * np.abs(ref)
    assert not np.isnan(got).any(), f"{what}: NaN"
    assert not bad.any(), f"{what}: {bad.sum()} bad, max err {err.max():.3e}"


def _case(K, B, Hkv, Hq, D, S, Smax, seed, calls=2, sm_scale=0.0):
    gen = torch.Generator().manual_seed(seed)
    k = torch.randn(B, Hkv, Smax, D, generator=gen).to(torch.bfloat16)
    v = torch.randn(B, Hkv, Smax, D, generator=gen).to(torch.bfloat16)
    # unused capacity holds NaN: it must never reach the output
    k[:, :, S:] = float("nan")
    v[:, :, S:] = float("nan")
    att = K.Bf16Attention(batch=B, num_kv_heads=Hkv, num_q_heads=Hq, head_dim=D)
    kd, vd = k.cuda(), v.cuda()
    for c in range(calls):
        q = torch.randn(B, Hq, D, generator=gen).to(torch.bfloat16)
        got = att.attend(kd, vd, S, q.cuda(), sm_scale=sm_scale).cpu().numpy()
        ref = O.attention_bf16(synth.bf16_bits(k), synth.bf16_bits(v), synth.bf16_bits(q), S,
                               sm_scale=sm_scale if sm_scale > 0 else None)
        _close(got, ref, f"B={B} Hkv={Hkv} Hq={Hq} D={D} S={S} call {c}")
    assert att.check_device_status() == 0
    tickets = (4 * B * Hkv + 255) // 256 * 256
    assert not att.workspace[:256 + tickets].any(), "status word and tickets return to zero"


@pytest.mark.parametrize("B,Hkv,Hq,D,S,Smax", [
    (1, 1, 1, 128, 1, 1),          # one token
    (2, 2, 8, 64, 77, 80),         # ragged last tile, HPK 4, D 64
    (1, 3, 3, 128, 10, 64),        # MHA, three warps without tokens
    (2, 1, 4, 128, 300, 300),
    (2, 2, 16, 128, 1000, 1030),   # HPK 8: separate hi and lo blocks
    (3, 2, 4, 64, 4097, 4100),     # pairs split across CTAs
    (1, 1, 2, 128, 20000, 20001),  # one pair over every CTA
    (64, 8, 8, 128, 70, 72),       # many pairs per CTA
])
def test_bf16_decode_matches_the_oracle(kivi, B, Hkv, Hq, D, S, Smax):
    _case(kivi, B, Hkv, Hq, D, S, Smax, seed=S * 7 + B)


def test_bf16_decode_sm_scale(kivi):
    _case(kivi, 2, 2, 4, 128, 333, 340, seed=3, calls=1, sm_scale=0.3)


def test_bf16_decode_llama3_8b_shape_sampled(kivi):
    """The Llama-3-8B GQA shape at S = 8193 (B 16, 8 kv heads, 32 query heads),
    in the launch configuration the benchmark's bf16 sweep uses; rows sampled."""
    B, Hkv, Hq, D, S = 16, 8, 32, 128, 8193
    gen = torch.Generator(device="cuda").manual_seed(12)
    k = torch.randn(B, Hkv, S + 63, D, generator=gen, device="cuda").to(torch.bfloat16)
    v = torch.randn(B, Hkv, S + 63, D, generator=gen, device="cuda").to(torch.bfloat16)
    q = torch.randn(B, Hq, D, generator=gen, device="cuda").to(torch.bfloat16)
    att = kivi.Bf16Attention(batch=B, num_kv_heads=Hkv, num_q_heads=Hq, head_dim=D)
    got = att.attend(k, v, S, q).cpu().numpy()
    for b, kvh in [(0, 0), (7, 3), (15, 7)]:
        kb = synth.bf16_bits(k[b:b + 1, kvh:kvh + 1, :S].cpu())
        vb = synth.bf16_bits(v[b:b + 1, kvh:kvh + 1, :S].cpu())
        qb = synth.bf16_bits(q[b:b + 1, kvh * 4:kvh * 4 + 4].cpu())
        ref = O.attention_bf16(kb, vb, qb)
        _close(got[b:b + 1, kvh * 4:kvh * 4 + 4], ref, f"b={b} kvh={kvh}")
    assert att.check_device_status() == 0
